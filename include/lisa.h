/*
 * lisa.h -- C ABI of the LISA (Linear-Indexed Sparse Attention) layer for
 * NVIDIA B200 (sm_100a).
 *
 * Method: "LISA: Linear-Indexed Sparse Attention for Efficient Long-Context
 * Reasoning" (arXiv 2607.19358).  Its abstract defines the layer: a Lightning
 * Indexer picks the top-M tokens of the whole context for a sparse softmax
 * self-attention, a linear-attention branch runs beside it, and a gate fuses
 * the two outputs, so n generated tokens cost O(nM).  The gptget.net digest of
 * the paper (section "方法详解", method details) adds: phi = identity with a
 * state matrix S_t, an indexer made of query/key projections and a ReLU dot
 * product, and a learned gate g; its "实验设计" (experiment design) section
 * gives M = 256.
 *
 * Definitions this library fixes where the pages are silent (the oracle used
 * by the tests applies the same ones):
 *   score   I_g(t,s) = sum_{r<R} w[t, g*R+r] * max(0, qidx[t, g*R+r] . kidx[g, s]),
 *           R = HI / Hkv, candidates s = 0..t (the current token included);
 *   select  per KV head g the first min(M, t+1) positions in the order
 *           (score descending, position ascending); -0.0 equals +0.0;
 *   sparse  o_sp[h] = softmax_{s in Sel_g}(q_h . k_s / sqrt(d)) . v_s for each
 *           query head h of group g = h / (Hq / Hkv);
 *   linear  S_h <- S_h + k_t^T v_t, then o_lin[h] = q_h S_h (no normaliser);
 *   gate    g = 1 / (1 + exp(-lambda_h)), o = g * o_sp + (1 - g) * o_lin.
 *
 * Conventions for every entry point
 *   - All tensor arguments are DEVICE pointers to dense row-major arrays owned
 *     by the caller, with one exception: the per-step inputs and outputs of
 *     lisa_decode_step (q, k, v, kidx, qidx, w, gate_logit, out, idx_out) may
 *     also be page-locked host memory mapped into the device's address space
 *     (cudaHostAlloc / cudaHostRegister with unified addressing, as torch's
 *     pin_memory() gives); the kernel then reads and writes them across the
 *     host link.  The layer's caches, state, pos and err_word, and every
 *     workspace, must be device memory.  The library never allocates, frees
 *     or synchronises.
 *   - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL =
 *     legacy default stream) and returns immediately.
 *   - Arguments are validated on the host before anything is launched; on
 *     failure nothing is launched and a status other than LISA_OK is returned.
 *     lisa_last_error_msg() then describes the failure (thread-local).
 *   - Launch failures reported by the CUDA runtime map to LISA_ERR_CUDA.
 *   - Checks that need device data (pos[b] out of range) are made on the
 *     device: the kernels skip the affected sequence and OR a bit into
 *     *err_word (when err_word is non-NULL); they never trap.  A call is
 *     asynchronous, so a status returned by the call can only describe what
 *     the host saw; everything found on the device (a bad position, a bounded
 *     wait that ran out, a failed self-check) is reported through these bits,
 *     which the caller reads after synchronising.
 *   - Every mbarrier wait inside a kernel (on an asynchronous copy, on another
 *     warp's progress, or on the messages of the other CTAs of a decode
 *     cluster) is bounded in time (LISA_WAIT_LIMIT_NS per wait, measured with
 *     the GPU's global nanosecond timer); a wait that runs out sets
 *     LISA_DEVERR_TIMEOUT and the kernel carries on to its end without
 *     waiting again for that stage.  Cluster barriers have no bounded form:
 *     every CTA of a cluster takes the same sequence of them.
 *   - Storage dtype (q, k, v, caches, out): bf16 or fp32, per lisa_layer.dtype.
 *     w, gate logits and the state are always fp32; indices are int32.
 *   - Supported shapes: d in {64, 128}; dI in {32, 64}; M a multiple of 32 in
 *     [32, 1024]; Hq % Hkv == 0, HI % Hkv == 0, HI / Hkv <= 8, Hq / Hkv <= 16;
 *     L_max >= 1.  Anything else returns LISA_ERR_UNSUPPORTED.
 *   - All pointers must be 16-byte aligned.
 */
#ifndef LISA_H_
#define LISA_H_

#include <stddef.h>

#if defined(__GNUC__)
#define LISA_API __attribute__((visibility("default")))
#else
#define LISA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LISA_OK = 0,
  LISA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, misaligned pointer */
  LISA_ERR_UNSUPPORTED = 2,   /* valid but outside the supported shapes */
  LISA_ERR_CUDA = 3,          /* the CUDA runtime rejected a launch */
  LISA_ERR_WORKSPACE = 4      /* workspace NULL or smaller than lisa_workspace_bytes() */
} lisa_status;

typedef enum { LISA_BF16 = 0, LISA_FP32 = 1 } lisa_dtype;

/* Bits a kernel ORs into *err_word. */
#define LISA_DEVERR_POS      1   /* pos[b] < 0, or pos[b] + T > L_max: sequence b skipped */
#define LISA_DEVERR_TIMEOUT  2   /* a bounded wait on an asynchronous copy gave up */
#define LISA_DEVERR_CHECK    4   /* an internal consistency check failed (a selected index out of
                                    range, or no threshold bucket); the access was skipped */

/* Time limit of one bounded wait inside a kernel, in nanoseconds. */
#define LISA_WAIT_LIMIT_NS   100000000ull

/* Bits of lisa_layer.debug_flags (testing the failure path; 0 in normal use). */
#define LISA_DEBUG_FORCE_TIMEOUT 1   /* lisa_decode_step: every CTA makes its first bounded wait on a
                                        barrier that no copy will complete, with a limit of 20
                                        microseconds, BEFORE issuing any copy; the wait runs out,
                                        LISA_DEVERR_TIMEOUT is ORed into err_word, and every CTA
                                        returns with nothing in flight.  Nothing else is written. */

/* Operation codes for lisa_workspace_bytes(). */
#define LISA_OP_DECODE       0
#define LISA_OP_PREFILL      1
#define LISA_OP_INDEXER_TOPK 2
#define LISA_OP_PREFILL_WINDOW 3

/* One attention layer: geometry plus the caller-owned per-layer buffers. */
typedef struct {
  int B;        /* sequences in the batch */
  int Hq;       /* query heads */
  int Hkv;      /* key/value heads; G = Hq / Hkv query heads share one */
  int d;        /* head dim of q, k, v */
  int HI;       /* indexer heads; R = HI / Hkv belong to each KV head */
  int dI;       /* indexer head dim */
  int M;        /* tokens kept per KV head by the top-M selection */
  int L_max;    /* rows of every cache buffer */
  int dtype;    /* lisa_dtype of q, k, v, caches and outputs */
  void *k_cache;     /* [B, Hkv, L_max, d]  */
  void *v_cache;     /* [B, Hkv, L_max, d]  */
  void *kidx_cache;  /* [B, Hkv, L_max, dI] indexer keys, one per KV head */
  float *state;      /* [B, Hq, d, d] fp32 linear state S[i][j] (key dim i, value dim j),
                        updated in place */
  const int *pos;    /* [B] device: position of the first new token of this call
                        (= tokens already cached) */
  int *err_word;     /* device int or NULL: LISA_DEVERR_* bits are ORed in */
  int decode_split;  /* CTAs that share one (sequence, KV head) in lisa_decode_step:
                        4, 8, 16: one thread-block cluster of that size (16 falls
                        back to 8 where 16-CTA clusters cannot be scheduled, 4 to
                        8 where its shared memory would not fit);
                        32, 64: the wide form, that many CTAs in clusters of 8
                        (bf16 storage and the decode workspace required; the
                        window and variant forms use 16 instead);
                        0: the library's choice: 16 when all 16-CTA clusters
                        fit on the device at once, else 8 or 4 (never the wide
                        form).  16 gives the shortest single step; 4 the least
                        SM time per step when many steps run concurrently.
                        Results do not depend on it beyond float summation
                        order.  Other calls ignore it. */
  int independent;   /* lisa_decode_step only.  0 (default): the step waits until the
                        launch before it on the stream has finished before it touches
                        memory (it is launched with programmatic dependent launch, so
                        only its start-up overlaps that launch).  1: the caller
                        declares that this call reads nothing the previous launch on
                        the stream writes, and writes nothing that launch reads or
                        writes (for example steps of independent layers or sequences
                        interleaved on one stream); the step then does not wait for
                        it and consecutive steps run concurrently on the device.
                        A wrong declaration gives wrong results, not an error. */
  int debug_flags;   /* LISA_DEBUG_* bits; 0 in normal use */
} lisa_layer;

/*
 * Bytes of scratch the caller must pass as `workspace` for operation `op`
 * (LISA_OP_*) with T new tokens per sequence.  Returns 0 for invalid input.
 * The workspace holds no state between calls (each call initialises what it
 * uses) but one workspace must not be used by two calls that overlap on the
 * device.
 */
LISA_API size_t lisa_workspace_bytes(const lisa_layer *layer, int T, int op);

/*
 * Append T new tokens per sequence to the caches (the cache write that
 * generating a token implies; abstract of arXiv 2607.19358).
 *   k, v  [B, T, Hkv, d]; kidx [B, T, Hkv, dI]   (storage dtype)
 * Row tau of sequence b goes to cache row pos[b] + tau.  Re-appending at the
 * same positions rewrites the same rows.  pos is not advanced.
 */
LISA_API lisa_status lisa_append_cache(const lisa_layer *layer, const void *k, const void *v,
                              const void *kidx, int T, void *stream);

/*
 * Lightning Indexer + top-M only (abstract of arXiv 2607.19358; score and order
 * as defined above) for T query tokens per sequence at positions
 * pos[b] .. pos[b]+T-1, against cache rows 0 .. pos[b]+tau (the caller must
 * have appended the T tokens first).
 *   qidx    [B, T, HI, dI] (storage dtype); w [B, T, HI] fp32
 *   idx_out [B, T, Hkv, M] int32: selected positions in ascending order,
 *           padded with -1 when the prefix holds fewer than M tokens.
 */
LISA_API lisa_status lisa_indexer_topk(const lisa_layer *layer, const void *qidx, const float *w, int T,
                              int *idx_out, void *workspace, size_t ws_bytes, void *stream);

/*
 * One decode step: the new token of every sequence sits at position t = pos[b].
 *   q [B, Hq, d]; k, v [B, Hkv, d]; kidx [B, Hkv, dI]; qidx [B, HI, dI]
 *   (storage dtype); w [B, HI] fp32; gate_logit [B, Hq] fp32
 *   out [B, Hq, d] (storage dtype)
 *   idx_out: NULL or [B, Hkv, M] int32 (the selected positions)
 * The new token's k, v, kidx are taken from the arguments (not the cache) and,
 * when fuse_append != 0, also written to cache row t.  With fuse_append == 0
 * the caller must already have stored them there.  The state is updated in
 * place (S <- S + k^T v).  pos is not advanced.
 * Forms (lisa_layer.decode_split).  In the cluster forms the indexer keys of
 * one (sequence, KV head) live in the shared memory of one thread-block
 * cluster, which bounds L_max to about 280K tokens (LISA_ERR_UNSUPPORTED
 * beyond); `workspace` is not used and may be NULL.  The wide form spreads
 * the key stream and the state of one (sequence, KV head) over 32 or 64 CTAs,
 * which publish their order keys and partial readouts of the linear branch
 * in the workspace; the last of their clusters to finish selects, attends
 * and writes the outputs.  It needs
 * lisa_workspace_bytes(layer, 1, LISA_OP_DECODE) bytes of workspace (0 for
 * fp32 storage, where the wide form does not apply), zero-filled before its
 * first use; every call leaves the workspace ready for the next one (its
 * arrival counters return to zero).  Calls that may run at the same time on
 * the device (steps declared independent, or steps on different streams)
 * need workspaces of their own.
 */
LISA_API lisa_status lisa_decode_step(const lisa_layer *layer, const void *q, const void *k, const void *v,
                             const void *kidx, const void *qidx, const float *w,
                             const float *gate_logit, int fuse_append, void *out, int *idx_out,
                             void *workspace, size_t ws_bytes, void *stream);

/*
 * Causal prefill of T tokens per sequence starting from an empty cache
 * (pos[b] must be 0; a sequence with another pos is skipped and flagged).
 *   q [B, T, Hq, d]; k, v [B, T, Hkv, d]; kidx [B, T, Hkv, dI];
 *   qidx [B, T, HI, dI] (storage dtype); w [B, T, HI] fp32;
 *   gate_logit [B, T, Hq] fp32; out [B, T, Hq, d] (storage dtype);
 *   idx_out: NULL or [B, T, Hkv, M] int32.
 * The T tokens are appended to the caches.  The state is read as S_0 and
 * overwritten with S_T.  Row tau's output equals the decode step of token tau.
 */
LISA_API lisa_status lisa_prefill(const lisa_layer *layer, int T, const void *q, const void *k,
                         const void *v, const void *kidx, const void *qidx, const float *w,
                         const float *gate_logit, void *out, int *idx_out, void *workspace,
                         size_t ws_bytes, void *stream);

/*
 * Stage-2 indexer objective, forward (arXiv 2607.19358, English abstract on
 * arxivdaily.com: the Indexer is trained with a per-head KL divergence that
 * aligns its selection with the frozen teacher's attention pattern).  For the
 * T tokens per sequence at positions t = pos[b] + tau and every query head h
 * (KV head g = h / G):
 *   p(s) = softmax over s <= t of q[b,tau,h] . k_cache[b,g,s] / sqrt(d)
 *   r(s) = softmax over s <= t of I_g(t, s)   (the indexer score defined above)
 *   kl_out[b, tau, h] = sum_s p(s) * (log p(s) - log r(s))      (fp32, >= 0)
 * The caches must already hold rows 0 .. pos[b]+T-1 (for example after
 * lisa_prefill or lisa_append_cache).  q [B, T, Hq, d]; qidx [B, T, HI, dI]
 * (bf16 storage only; LISA_ERR_UNSUPPORTED otherwise); w [B, T, HI] fp32;
 * kl_out [B, T, Hq] fp32.  No workspace.
 */
LISA_API lisa_status lisa_indexer_kl(const lisa_layer *layer, int T, const void *q, const void *qidx,
                                     const float *w, float *kl_out, void *stream);

/*
 * Stage-1 inference variant: sliding window (arXiv 2607.19358, English
 * abstract on arxivdaily.com: Stage 1 pairs the linear attention with a
 * sliding-window attention, which Stage 2 replaces by the Lightning Indexer;
 * iitog.ru article, key facts).  The sparse branch attends to the M most
 * recent positions max(0, t-M+1) .. t (the layer's M is the window); the
 * linear branch, the gate and every other definition are those of
 * lisa_decode_step / lisa_prefill.  No indexer inputs: kidx may be NULL (the
 * indexer-key cache row is then not written); qidx and w are not taken.
 * idx_out, when given, receives the window's positions ([B, Hkv, M] for the
 * step, [B, T, Hkv, M] for the prefill; ascending, -1 padded).  The decode
 * step needs no workspace; the prefill needs
 * lisa_workspace_bytes(layer, T, LISA_OP_PREFILL_WINDOW).
 */
LISA_API lisa_status lisa_decode_step_window(const lisa_layer *layer, const void *q, const void *k, const void *v,
                                             const void *kidx, const float *gate_logit, int fuse_append,
                                             void *out, int *idx_out, void *stream);
LISA_API lisa_status lisa_prefill_window(const lisa_layer *layer, int T, const void *q, const void *k,
                                         const void *v, const void *kidx, const float *gate_logit, void *out,
                                         int *idx_out, void *workspace, size_t ws_bytes, void *stream);

/*
 * lisa_indexer_topk without a workspace argument, for callers that cannot
 * allocate device memory: for example a plugin running inside a host program
 * that owns all device memory and gives the plugin no allocator, or code that
 * may not call cudaMalloc because it can synchronise the device.  The method's
 * pages have no counterpart for this call; it is a convenience of this library.
 *
 * Arguments, results and checks are those of lisa_indexer_topk.  The scratch
 * comes from one fixed array of LISA_NOALLOC_SCRATCH_BYTES in device memory
 * that every GPU which loads the library holds until the process exits.  A
 * call needs B * Hkv * L_max * 4 bytes (L_max rounded up to a multiple of 4)
 * of it per query row: larger sizes return LISA_ERR_UNSUPPORTED before
 * anything is launched, and smaller ones process the T rows in as many passes
 * as the array requires.  The call allocates and frees nothing.
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it; make that first call before any stream
 * capture.  All calls share the one array and it keeps the last call's
 * contents (nothing in it needs to start at zero: every entry a call reads it
 * has written first).  Calls that overlap on the GPU, from any stream or
 * thread, race on the array and must be avoided.
 */
#define LISA_NOALLOC_SCRATCH_BYTES (16u << 20)
LISA_API lisa_status lisa_indexer_topk_noalloc(const lisa_layer *layer, const void *qidx, const float *w,
                                               int T, int *idx_out, void *stream);

/*
 * Definition variants of the head mapping.  The pages say only that the
 * indexer is a ReLU dot product of small query/key projections (gptget.net
 * digest, method details) and that a linear-attention branch with phi =
 * identity runs beside the sparse attention (abstract); how indexer heads,
 * indexer keys and the linear branch's keys and values map onto the attention
 * heads is left open.  The calls above fix one reading (one indexer key per KV
 * head, one top-M set per KV head, the attention's own k and v in the linear
 * branch).  These flags select the other readings:
 *
 *   LISA_VAR_KEY_PER_INDEXER_HEAD   every indexer head j has a key of its own:
 *       I_g(t,s) = sum_{r<R} w[t,j] * max(0, qidx[t,j] . kidx[j, s]), j = g*R + r.
 *       The indexer-key cache and the new tokens' kidx hold HI planes.
 *   LISA_VAR_SHARED_SET             one top-M set per token, shared by every
 *       KV head (Gs = 1 selection group over all HI indexer heads):
 *       I(t,s) = sum_{j<HI} w[t,j] * max(0, qidx[t,j] . kidx[p(j), s]) with
 *       p(j) = j under KEY_PER_INDEXER_HEAD and p(j) = 0 (one key per token)
 *       otherwise.  Index lists have one group instead of Hkv.
 *   LISA_VAR_LINEAR_KV_PER_QUERY_HEAD  the linear branch takes keys and
 *       values of its own for every query head: S_h <- S_h + k_lin[h]^T
 *       v_lin[h] (k_lin, v_lin [B, (T,) Hq, d], storage dtype).
 *
 * Shapes under a variant (P = indexer-key planes, Gs = selection groups):
 *   P  = HI with KEY_PER_INDEXER_HEAD, else 1 with SHARED_SET, else Hkv;
 *   Gs = 1 with SHARED_SET, else Hkv.
 * The layer's kidx_cache is then [B, P, L_max, dI] and kidx arguments are
 * [B, (T,) P, dI]; idx_out is [B, (T,) Gs, M].  Everything else (selection
 * order, softmax scale, gate, state layout) is as defined at the top.
 * variant = 0 is the default reading and runs the same kernels as the calls
 * above.  With KEY_PER_INDEXER_HEAD or SHARED_SET the decode step runs the
 * indexer and top-M through the row path (scores in the workspace) before the
 * attention kernel, so it needs
 * lisa_workspace_bytes_variant(layer, variant, 1, LISA_OP_DECODE) bytes of
 * workspace; the prefill needs lisa_workspace_bytes_variant(layer, variant, T,
 * LISA_OP_PREFILL).  Unknown flag bits return LISA_ERR_INVALID_ARG; k_lin and
 * v_lin are required with LINEAR_KV_PER_QUERY_HEAD and ignored otherwise.
 */
#define LISA_VAR_KEY_PER_INDEXER_HEAD     1
#define LISA_VAR_SHARED_SET               2
#define LISA_VAR_LINEAR_KV_PER_QUERY_HEAD 4

LISA_API size_t lisa_workspace_bytes_variant(const lisa_layer *layer, int variant, int T, int op);
/* lisa_append_cache with kidx [B, T, P, dI] (P planes of the variant). */
LISA_API lisa_status lisa_append_cache_variant(const lisa_layer *layer, int variant, const void *k, const void *v,
                                               const void *kidx, int T, void *stream);
/* lisa_indexer_topk under a variant; idx_out [B, T, Gs, M]; workspace
 * lisa_workspace_bytes_variant(layer, variant, T, LISA_OP_INDEXER_TOPK). */
LISA_API lisa_status lisa_indexer_topk_variant(const lisa_layer *layer, int variant, const void *qidx,
                                               const float *w, int T, int *idx_out, void *workspace,
                                               size_t ws_bytes, void *stream);
/* lisa_decode_step under a variant: kidx [B, P, dI]; k_lin, v_lin [B, Hq, d];
 * idx_out NULL or [B, Gs, M]. */
LISA_API lisa_status lisa_decode_step_variant(const lisa_layer *layer, int variant, const void *q, const void *k,
                                              const void *v, const void *kidx, const void *qidx, const float *w,
                                              const float *gate_logit, const void *k_lin, const void *v_lin,
                                              int fuse_append, void *out, int *idx_out, void *workspace,
                                              size_t ws_bytes, void *stream);
/* lisa_prefill under a variant: kidx [B, T, P, dI]; k_lin, v_lin [B, T, Hq, d];
 * idx_out NULL or [B, T, Gs, M]. */
LISA_API lisa_status lisa_prefill_variant(const lisa_layer *layer, int variant, int T, const void *q,
                                          const void *k, const void *v, const void *kidx, const void *qidx,
                                          const float *w, const float *gate_logit, const void *k_lin,
                                          const void *v_lin, void *out, int *idx_out, void *workspace,
                                          size_t ws_bytes, void *stream);

/*
 * Projections on either side of the layer (abstract and gptget.net digest,
 * method details: the attention's q, k, v, the indexer's query / key
 * projections, its head weights and the gate are projections of the hidden
 * state; the layer's output returns to the hidden size).  The pages give no
 * fused form; this library reads the front-end as ONE linear map of the
 * hidden state x [Hm] whose output columns are, in this order,
 *   q [Hq*d] | k [Hkv*d] | v [Hkv*d] | qidx [HI*dI] | kidx [P*dI] | w [HI] | gate_logit [Hq]
 * (P indexer-key planes as for the variants above; Hkv by default), and the
 * output projection as y = o W_o^T.  Weights are stored out-features x
 * in-features, bf16: W_in [N_in, Hm] with N_in the sum of the widths above,
 * W_o [Hm, Hq*d].  Accumulation is fp32 on the tensor cores; w and gate_logit
 * are written in fp32, everything else in bf16.  bf16 storage only
 * (LISA_ERR_UNSUPPORTED otherwise); Hm a multiple of 8.
 */
typedef struct {
  int Hm;              /* hidden size */
  const void *W_in;    /* [N_in, Hm] bf16 */
  const void *W_o;     /* [Hm, Hq * d] bf16 */
} lisa_proj;

/* Front-end for T tokens per sequence: x [B, T, Hm] -> q [B, T, Hq, d],
 * k, v [B, T, Hkv, d], qidx [B, T, HI, dI], kidx [B, T, P, dI] (bf16),
 * w [B, T, HI], gate_logit [B, T, Hq] (fp32): the inputs of lisa_prefill /
 * lisa_decode_step (T = 1) and their _variant forms.  variant only sets P. */
LISA_API lisa_status lisa_project_in(const lisa_layer *layer, int variant, const lisa_proj *proj, int T,
                                     const void *x, void *q, void *k, void *v, void *qidx, void *kidx, float *w,
                                     float *gate_logit, void *stream);
/* Output projection for T tokens per sequence: o [B, T, Hq, d] -> y [B, T, Hm] (bf16). */
LISA_API lisa_status lisa_project_out(const lisa_layer *layer, const lisa_proj *proj, int T, const void *o,
                                      void *y, void *stream);

/* Human-readable name of a status. */
LISA_API const char *lisa_status_str(lisa_status s);

/* Description of the last failure on the calling thread ("" if none). */
LISA_API const char *lisa_last_error_msg(void);

/* Library version string. */
LISA_API const char *lisa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LISA_H_ */
