/*
 * hils.h -- C ABI of libhils.so: the forward pass of HiLS (Hierarchical
 * Landmark Sparse) attention on NVIDIA B200 (sm_100a).
 *
 * The method (pages on "Hierarchical Sparse Attention Done Right: Toward
 * Infinite Context Modeling"):
 *   - model card "HiLS-Attention" (axforge.ai), section "What HiLS-Attention
 *     is": one compressed (landmark) key per chunk estimates the chunk's mass;
 *     attention factorises into an inter-chunk and an intra-chunk softmax; the
 *     top-k chunks are selected;
 *   - molayo1419.me article, section "Core idea": step 1, inter-chunk
 *     attention of the query over all landmark keys; step 2, standard
 *     attention inside the selected chunks;
 *   - aiweekly.co article, mechanism paragraph: each query attends to each
 *     retrieved chunk independently and the outputs are fused by the chunk
 *     retrieval scores;
 *   - molayo1419.me article, section "Hardware-efficient kernel": M adjacent
 *     queries share the union of their chunks, loaded once.
 *
 * Conventions shared by every call
 *   Layout: BHLD, contiguous.  q [B,Hq,L,d], k and v [B,Hkv,L,d], landmark
 *   keys lmk_k [B,Hkv,floor(L/C),d] (one per complete chunk).  Query head hq
 *   reads KV head hq / (Hq/Hkv).  Element type of q, k, v, lmk_k and out is
 *   params.dtype (fp32 or bf16); chunk_w, lse_lmk, lse and w_final are fp32;
 *   sel_idx is int32.
 *   Row t (0-based) has own chunk floor(t/C) and completed chunks
 *   c < floor(t/C).  Its own chunk is always attended, causally (keys <= t),
 *   with fusion logit equal to the log-sum-exp of its causal token logits;
 *   it does not take a top-k slot.  Selection order is (landmark logit
 *   descending, chunk index ascending); rows with fewer than k completed
 *   chunks select all of them.  The fusion weights are a softmax over the
 *   selected landmark logits plus the own-chunk logit.
 *   Pointers: every array argument is a DEVICE pointer owned by the caller,
 *   16-byte aligned.  The library allocates no device memory and keeps no
 *   state other than cached device attributes, a launch counter and the
 *   fixed scratch array of hils_decode_fwd_noalloc (module memory, below).
 *   Streams: every call is asynchronous on `stream` (a cudaStream_t passed as
 *   void*; NULL = legacy default stream) and ordered on it as a whole: a
 *   call's first kernel starts after the work queued before it, and work
 *   queued after it starts after its last kernel (inside a decode call the
 *   kernels after the first overlap their predecessors' ends through
 *   programmatic dependent launch).  Argument and shape errors are
 *   returned before anything is launched.  A launch failure returns
 *   HILS_ERR_CUDA.  With params.debug_checks = 1 the call also validates its
 *   selections on the device and synchronises the stream to report
 *   HILS_ERR_DEVICE_CHECK (a bad index) or HILS_ERR_TIMEOUT (a bounded
 *   device wait gave up); device code never traps.
 *   Supported: dtype bf16 with d in {64, 128}, or fp32 with d in {64, 128};
 *   chunk C = 64; 1 <= topk <= 64; Hq % Hkv == 0; M in {16, 32, 64, 128};
 *   L >= 1 (a ragged last chunk is allowed; it is never complete).  Anything
 *   else returns HILS_ERR_UNSUPPORTED.
 */
#ifndef HILS_H_
#define HILS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HILS_OK = 0,
  HILS_ERR_INVALID_ARG = 1, /* null pointer, misaligned pointer, bad shape */
  HILS_ERR_UNSUPPORTED = 2, /* valid but not implemented (dtype, d, chunk...) */
  HILS_ERR_WORKSPACE = 3,   /* ws too small (see hils_workspace_size) */
  HILS_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
  HILS_ERR_DEVICE_CHECK = 5,/* debug_checks: a device-side check failed */
  HILS_ERR_TIMEOUT = 6      /* debug_checks: a bounded device wait gave up */
} hils_status;

typedef enum { HILS_F32 = 0, HILS_BF16 = 1 } hils_dtype;

typedef struct {
  int B, Hq, Hkv; /* batch, query heads, KV heads (Hq % Hkv == 0) */
  int L;          /* prefill: sequence length; decode: KV-cache length N,
                     which already includes the new token (query at N-1) */
  int d;          /* head dimension */
  int chunk;      /* C, tokens per chunk */
  int topk;       /* k, chunks selected per query */
  int M;          /* adjacent queries per group of hils_union (16, 32, 64
                     or 128).  The prefill kernels do not read it: they
                     always load the union of a 128-row tile (the tensor
                     core's full-rate M), so their results do not depend
                     on it */
  float scale;    /* softmax scale of token and landmark logits (1/sqrt(d)) */
  int dtype;      /* hils_dtype of q, k, v, lmk_k and out */
  int debug_checks; /* 0 or 1, see above */
} hils_params;

#define HILS_OP_PREFILL 0
#define HILS_OP_DECODE 1

/* Bytes of device workspace `op` needs for these params (0 is possible).
 * Returns 0 for invalid params as well; the calls themselves validate. */
size_t hils_workspace_size(const hils_params *p, int op);

/*
 * Landmark scoring, inter-chunk softmax normaliser and top-k selection
 * (model card, "What HiLS-Attention is"; molayo1419.me, "Core idea", step 1).
 *   q       [B,Hq,L,d]          in
 *   lmk_k   [B,Hkv,L/C,d]       in
 *   sel_idx [B,Hq,L,topk] int32 out: selected chunk ids, ascending, -1 pad
 *   chunk_w [B,Hq,L,topk] fp32  out: their landmark logits
 *                                    scale*<q_t, lmk_c>, -inf pad
 *   lse_lmk [B,Hq,L] fp32       out, may be NULL: log-sum-exp of the logits of
 *                                    all completed chunks (-inf if none); the
 *                                    inter-chunk softmax is exp(chunk_w - lse_lmk)
 */
hils_status hils_select(const hils_params *p, const void *q, const void *lmk_k,
                        int32_t *sel_idx, float *chunk_w, float *lse_lmk,
                        void *ws, size_t ws_bytes, void *stream);

/*
 * Chunk union per group of M adjacent queries (molayo1419.me, "Hardware-
 * efficient kernel"): for group g = [g*M, (g+1)*M) of head (b, hq), the
 * ascending set of all chunk ids selected by its rows plus each row's own
 * chunk, in CSR form.  Groups are ordered (b, hq, g); G = B*Hq*ceil(L/M).
 *   sel_idx [B,Hq,L,topk] int32 in (as written by hils_select)
 *   u_off   [G+1] int32         out: u_off[0] = 0, u_off[G] = total
 *   u_idx   [u_cap] int32       out: concatenated sets
 *   u_cap   capacity of u_idx; must be >= hils_union_capacity(p)
 * hils_attn_fwd does not need this output: it builds each tile's union
 * internally.  This call materialises it (union-size statistics, checks).
 */
int64_t hils_union_capacity(const hils_params *p);
hils_status hils_union(const hils_params *p, const int32_t *sel_idx, int32_t *u_off,
                       int32_t *u_idx, int64_t u_cap, void *ws, size_t ws_bytes,
                       void *stream);

/*
 * Intra-chunk attention over the selected chunks and the own chunk, and
 * score-weighted fusion (molayo1419.me, "Core idea", step 2; aiweekly.co,
 * mechanism paragraph).
 *   q, k, v  in (see layout)
 *   sel_idx, chunk_w  in: a selection as written by hils_select (ascending
 *            ids, -1 pad; logits of the selected chunks)
 *   out      [B,Hq,L,d] dtype out
 *   lse      [B,Hq,L] fp32 out: log-sum-exp of the fused chunk logits
 *   w_final  [B,Hq,L,topk+1] fp32 out, may be NULL: fusion weights of the
 *            selected chunks in sel_idx order (0 for padding), own chunk last
 */
hils_status hils_attn_fwd(const hils_params *p, const void *q, const void *k, const void *v,
                          const int32_t *sel_idx, const float *chunk_w, void *out,
                          float *lse, float *w_final, void *ws, size_t ws_bytes,
                          void *stream);

/* hils_select followed by hils_attn_fwd on the same stream. */
hils_status hils_prefill(const hils_params *p, const void *q, const void *k, const void *v,
                         const void *lmk_k, int32_t *sel_idx, float *chunk_w, float *lse_lmk,
                         void *out, float *lse, void *ws, size_t ws_bytes, void *stream);

/*
 * One decode step for B sequences (prefill of a single row t = N-1 per head,
 * with the KV cache already holding the new token).
 *   q        [B,Hq,d]          in
 *   k_cache, v_cache [B,Hkv,N,d] in (N = p->L)
 *   lmk_k    [B,Hkv,N/C,d]     in
 *   sel_idx  [B,Hq,topk] int32 out, chunk_w [B,Hq,topk] fp32 out,
 *   lse_lmk  [B,Hq] fp32 out (may be NULL), out [B,Hq,d] dtype out,
 *   lse      [B,Hq] fp32 out
 * Needs hils_workspace_size(p, HILS_OP_DECODE) bytes of workspace.
 */
hils_status hils_decode_fwd(const hils_params *p, const void *q, const void *k_cache,
                            const void *v_cache, const void *lmk_k, int32_t *sel_idx,
                            float *chunk_w, float *lse_lmk, void *out, float *lse, void *ws,
                            size_t ws_bytes, void *stream);

/*
 * The decode step of hils_decode_fwd over a paged KV cache, the form an
 * inference engine's attention backend is handed (molayo1419.me, "Converting
 * existing models": serving runs HiLS as an attention backend of an SGLang
 * fork; the page layout below is this library's).  A page holds one chunk
 * (C = p->chunk tokens) of every KV head:
 *   k_pages, v_pages [num_pages, Hkv, C, d] in (dtype), both of num_pages
 *            pages; a page of a partial last chunk holds its
 *            N - C*(ceil(N/C)-1) tokens first
 *   page_table [B, max_pages_per_seq] int32 in (device): page of chunk c of
 *            sequence b; entries c < ceil(N/C) are read, the rest ignored
 *   lmk_k    [B,Hkv,N/C,d] in: the landmark keys stay a dense per-sequence
 *            array (one row per chunk, 1/C of the cache)
 * Everything else (q, outputs, workspace, N = p->L) is as in hils_decode_fwd;
 * the results equal hils_decode_fwd on the dense caches the table describes.
 * Pages may be shared or in any order.  An entry outside [0, num_pages) is
 * never dereferenced: that chunk's attention output is unspecified and, with
 * p->debug_checks, the call returns HILS_ERR_DEVICE_CHECK.
 */
hils_status hils_decode_fwd_paged(const hils_params *p, const void *q, const void *k_pages,
                                  const void *v_pages, int64_t num_pages,
                                  const int32_t *page_table, int max_pages_per_seq,
                                  const void *lmk_k, int32_t *sel_idx, float *chunk_w,
                                  float *lse_lmk, void *out, float *lse, void *ws,
                                  size_t ws_bytes, void *stream);

/*
 * Allocation-free variant of hils_decode_fwd.  The paper has no counterpart:
 * this is a deployment aid.  It is for callers that cannot pass a workspace
 * because they cannot allocate device memory -- e.g. a serving framework that
 * reserves all GPU memory for its own pool and forbids cudaMalloc elsewhere,
 * or a per-token decode loop where cudaMalloc/cudaFree would synchronise the
 * device.  Arguments and results are those of hils_decode_fwd, without ws.
 * The decode scratch lives in a fixed 32 MiB device array inside the library
 * (held on every GPU that loads the library until the process exits); shapes
 * that need more scratch return HILS_ERR_WORKSPACE before any launch.  The
 * first call on a device looks the array up (cudaGetSymbolAddress, which may
 * load the library's module there): make it before any stream capture.  The
 * address belongs to the device's context; after the context changes (e.g.
 * cudaDeviceReset) the next call looks it up again, so that call too should
 * come before any stream capture.  All
 * calls share the array and it keeps the last call's contents (each call
 * writes every scratch entry it reads); calls that overlap on the GPU race
 * and must be serialised by the caller.  Nothing here allocates.
 */
hils_status hils_decode_fwd_noalloc(const hils_params *p, const void *q, const void *k_cache,
                                    const void *v_cache, const void *lmk_k, int32_t *sel_idx,
                                    float *chunk_w, float *lse_lmk, void *out, float *lse,
                                    void *stream);

/*
 * Backward pass of the forward above (aiweekly.co, mechanism paragraph: the
 * chunk outputs are fused by the chunk scores, so the loss reaches them;
 * molayo1419.me, "Core idea": the landmark keys take part in the forward
 * pass).  The top-k choice carries no gradient: the forward's selection is an
 * input.  Gradients of sum(out * dout) + sum(lse * dlse) with respect to q, k,
 * v and the landmark keys:
 *   q, k, v, lmk_k     in, as for the forward (params dtype)
 *   sel_idx, chunk_w   in: the forward's selection and landmark logits
 *   lse  [B,Hq,L] fp32 in: the forward's lse
 *   dout [B,Hq,L,d]    in (params dtype); dlse [B,Hq,L] fp32 in, may be NULL (0)
 *   dq [B,Hq,L,d], dk, dv [B,Hkv,L,d], dlmk [B,Hkv,L/C,d]  fp32 out (every
 *   element written; dlmk may be NULL when L < C)
 *   ws >= hils_attn_bwd_workspace_size(p) bytes: per-(row, attended chunk)
 *   records of 16 bytes and the transposed selection (8 bytes per selected
 *   chunk of every row), plus 2 KB.
 * dk, dv and dlmk sum over the rows that attend a chunk in an order set by
 * atomic operations, so their last bits may differ from run to run; dq is
 * deterministic.  B*Hq*L*topk must be below 2^31.
 */
size_t hils_attn_bwd_workspace_size(const hils_params *p);
hils_status hils_attn_bwd(const hils_params *p, const void *q, const void *k, const void *v,
                          const void *lmk_k, const int32_t *sel_idx, const float *chunk_w,
                          const float *lse, const void *dout, const float *dlse, float *dq,
                          float *dk, float *dv, float *dlmk, void *ws, size_t ws_bytes,
                          void *stream);

/*
 * Q-Cal scoring query (molayo1419.me, "Engineering details", Q-Cal): a
 * low-rank learnable offset of the query, used only for the chunk scores.
 *   q_cal[b,hq,t,:] = q[b,hq,t,:] + W_up[hq] (W_down h[b,t,:])
 *   q       [B,Hq,L,d] in (params dtype)
 *   h       [B,L,D] in (params dtype): the token's hidden state
 *   w_down  [r,D] in (params dtype), shared by the heads
 *   w_up    [Hq,d,r] in (params dtype)
 *   q_cal   [B,Hq,L,d] out (params dtype), may not alias q
 *   1 <= r <= 64, D >= 1; ws >= hils_qcal_workspace_size(p, r) bytes
 *   (device scratch, B*L*r fp32 plus 256 bytes).
 * Arithmetic: fp32, each product and partial sum rounded separately (no
 * fused multiply-add), sums over D then over r in ascending order, and a bf16
 * query rounded to nearest even at the end -- the pages fix no precision, so
 * the query's own is used and the scoring pass sees exactly this query.
 * hils_select on q_cal gives the selection, the chunk logits and lse_lmk of
 * the calibrated scores; attention (hils_attn_fwd) keeps q.
 */
size_t hils_qcal_workspace_size(const hils_params *p, int r);
hils_status hils_qcal_query(const hils_params *p, const void *q, const void *h,
                            const void *w_down, const void *w_up, int D, int r, void *q_cal,
                            void *ws, size_t ws_bytes, void *stream);

/* hils_qcal_query, then hils_select on q_cal, then hils_attn_fwd on q, on
 * one stream.  q_cal [B,Hq,L,d] is the caller's scratch (the calibrated
 * query, left there). */
hils_status hils_prefill_qcal(const hils_params *p, const void *q, const void *k, const void *v,
                              const void *lmk_k, const void *h, const void *w_down,
                              const void *w_up, int D, int r, void *q_cal, int32_t *sel_idx,
                              float *chunk_w, float *lse_lmk, void *out, float *lse, void *ws,
                              size_t ws_bytes, void *stream);

/*
 * HoPE, the positional encoding of the pages (molayo1419.me, "Engineering
 * details", HoPE): rotary position embedding on the dimensions inside the
 * pre-training window, none (NoPE) on the rest.  Applied in place to q or k
 * before hils_prefill / hils_decode_fwd (a decode query at pos0 = N-1; keys
 * as they enter the cache); the landmark keys are left to the caller.
 *   x      [B, H, L, d] in/out, dtype HILS_F32 or HILS_BF16; row (b, h, t)
 *          has position pos0 + t
 *   n_rope_pairs  number of rotated pairs, 0..d/2: dimensions pair up as
 *          (i, i + d/2) and pair i < n_rope_pairs turns by the angle
 *          (pos0 + t) * base^(-2i/d); the other pairs are not touched.  The
 *          pages give no split rule: the caller picks it (e.g. the pairs
 *          whose wavelength 2*pi*base^(2i/d) fits the pre-training length)
 *   base   > 1
 * Asynchronous on `stream`; invalid arguments are refused before the launch.
 */
hils_status hils_hope(void *x, int dtype, int B, int H, int L, int d, int pos0,
                      int n_rope_pairs, double base, void *stream);

/*
 * Prefill with HoPE applied to the queries inside the kernels (bf16 only):
 * q is taken as it comes, unrotated, and each query tile is rotated as it is
 * staged -- in the scoring kernel on its way to tensor memory, in the
 * attention kernel in shared memory -- exactly as hils_hope(q, pos0,
 * n_rope_pairs, base) would rotate it (same arithmetic, same bits), so the
 * query pre-pass over HBM disappears.  k must hold keys already rotated, as
 * a cache does (hils_hope on the keys once, when they enter it); the
 * landmark keys are used as given.  Everything else is hils_prefill's.
 * fp32 parameters return HILS_ERR_UNSUPPORTED (rotate with hils_hope).
 */
hils_status hils_prefill_hope(const hils_params *p, const void *q, const void *k, const void *v,
                              const void *lmk_k, int pos0, int n_rope_pairs, double base,
                              int32_t *sel_idx, float *chunk_w, float *lse_lmk, void *out,
                              float *lse, void *ws, size_t ws_bytes, void *stream);

/*
 * The HoPE split (molayo1419.me, "Engineering details", HoPE: rotary
 * embedding on the dimensions inside the pre-training window, none beyond):
 * the number of rotate-half pairs i whose wavelength 2*pi*base^(2i/d) is at
 * most train_len, the pre-training length in tokens.  These are the pairs
 * 0 .. n-1 (the wavelength grows with i); pass n as n_rope_pairs.  Host
 * function, no GPU work; returns -1 for d < 2, base <= 1 or NaN arguments.
 */
int hils_hope_rope_pairs(int d, double base, double train_len);

/*
 * Failure-path testing only (not for production use).  Every device wait of
 * the prefill kernels (hils_select, hils_attn_fwd and the calls built on
 * them) is bounded: after ns nanoseconds (default 2 s; ns = 0 restores it)
 * the waiting role raises the kernel's abort flag, every role unwinds through
 * the common teardown (in-flight copies and tensor-core work are waited for,
 * tensor memory is freed) and, with params.debug_checks = 1, the call
 * returns HILS_ERR_TIMEOUT.  withhold = 1 makes the scoring kernel keep back
 * one arrival on its first landmark tile, so that such a wait runs out on
 * purpose; nothing faults, traps or waits without a bound.  Process-wide;
 * set it only while no other thread calls the library.
 */
void hils_test_set_wait_limit(uint64_t ns, int withhold);

/* Static description of a status code. */
const char *hils_status_string(hils_status s);

/* Human-readable detail of the last failure on the calling thread ("" if none). */
const char *hils_last_error(void);

/* Number of kernels this library has launched in this process so far. */
int64_t hils_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* HILS_H_ */
