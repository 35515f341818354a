"""Plain, slow, fp64 reference of the LISA attention layer.

TEST INFRASTRUCTURE ONLY: the CUDA library never imports or calls this module,
and this module imports nothing from the CUDA side.  Every function works on
float64 NumPy arrays and follows one step of the method in the order the pages
give it.

Sources (web pages about arXiv 2607.19358, "LISA: Linear-Indexed Sparse
Attention for Efficient Long-Context Reasoning"):
  [abs]  the English abstract (arxivdaily.com page; same text on fugumt.com):
         a Lightning Indexer keeps the top-M tokens of the full context for a
         sparse self-attention; a linear-attention branch runs in parallel;
         a gate fuses the two; n generated tokens cost O(nM).
  [meth] gptget.net digest, section "方法详解" (method details): linear
         attention with phi = identity and a state matrix S_t updated in O(1)
         per step; indexer = query/key projections and a ReLU dot product;
         a learned gate g mixes the two branch outputs.
  [exp]  gptget.net digest, section "实验设计" (experiment design): M = 256.

The pages leave these points open; this library fixes them as definitions
(the same in the oracle and on the GPU):
  * indexer score of key s for KV head g: sum over the R = HI/Hkv indexer heads
    j = g*R + r of w[j] * max(0, qidx[j] . kidx[g, s]); no extra scale;
  * one top-M set per KV head, shared by its G = Hq/Hkv query heads
    (query head h belongs to KV head h // G);
  * the other readings of the head mapping are variants behind keyword
    arguments: one indexer key per indexer head, a single top-M set shared by
    all KV heads, and linear-branch keys / values of their own per query head;
  * order: higher score first, equal scores -> lower position first;
    a prefix with <= M tokens is selected whole; the current token is a
    candidate (causal prefix s <= t);
  * softmax scale 1/sqrt(d);
  * linear branch: S_h <- S_h + k_t^T v_t, then o_lin = q_t S_h (the update
    includes the current token), no normaliser, no decay; k and v are the
    attention's own k/v of KV head h // G, S is kept per query head;
  * gate: g = sigmoid(lambda_h), o = g * o_sparse + (1 - g) * o_lin.

Parity status of each function is stated in its docstring; every function here
is pinned by tests in tests/test_oracle.py.
"""

import numpy as np


# --------------------------------------------------------------------------
# step 1: Lightning Indexer score      [abs], [meth]
# --------------------------------------------------------------------------
def indexer_scores(qidx_t: np.ndarray, w_t: np.ndarray, kidx_keys: np.ndarray, groups=None) -> np.ndarray:
    """Scores of every candidate key for one query token.

    qidx_t    [HI, dI]      indexer queries of the token
    w_t       [HI]          indexer head weights of the token
    kidx_keys [P, n, dI]    indexer keys of the candidate positions 0..n-1
    groups    selection groups Gs (default P): the HI heads are split into Gs
              groups of R = HI / Gs consecutive heads, one score row per group
    returns   [Gs, n]       I_gs(s) = sum_r w[j] * max(0, qidx[j] . key_j[s]),
                            j = gs*R + r

    key_j is plane gs when P == Gs (one indexer key per group: per KV head in
    the default reading, a single key per token for a shared selection) and
    plane j when P == HI (one indexer key per indexer head, the other reading
    of the head mapping the pages leave open).
    """
    HI = qidx_t.shape[0]
    P, n, _ = kidx_keys.shape
    Gs = P if groups is None else int(groups)
    R = HI // Gs
    assert Gs * R == HI and P in (Gs, HI), "key planes must be one per group or one per indexer head"
    out = np.zeros((Gs, n), dtype=np.float64)
    for gs in range(Gs):
        for r in range(R):
            j = gs * R + r
            plane = gs if P == Gs else j
            dots = kidx_keys[plane] @ qidx_t[j]
            out[gs] += w_t[j] * np.maximum(dots, 0.0)
    return out


# --------------------------------------------------------------------------
# step 2: top-M selection              [abs], [exp]
# --------------------------------------------------------------------------
def _order(scores: np.ndarray) -> np.ndarray:
    """Positions sorted by (score descending, position ascending)."""
    n = scores.shape[0]
    # np.lexsort sorts by the last key first: primary -score, secondary position.
    return np.lexsort((np.arange(n), -scores))


def topm_select(scores: np.ndarray, M: int) -> np.ndarray:
    """The first min(M, n) positions of the order, listed in ascending position,
    padded with -1 up to M entries."""
    n = scores.shape[0]
    keep = np.sort(_order(scores)[: min(M, n)])
    out = np.full(M, -1, dtype=np.int64)
    out[: keep.shape[0]] = keep
    return out


def window_select(t: int, W: int) -> np.ndarray:
    """Stage-1 inference variant (arxivdaily.com English abstract: Stage 1
    pairs the linear attention with a sliding-window attention that the
    Indexer later replaces; iitog.ru article, key facts): the sparse branch
    attends to the W most recent positions max(0, t-W+1) .. t, listed in
    ascending position, padded with -1 up to W entries.

    Parity: pinned against topm_select on scores that increase with the
    position (the top-W of such scores is the last W positions)."""
    lo = max(0, t - W + 1)
    out = np.full(W, -1, dtype=np.int64)
    keep = np.arange(lo, t + 1, dtype=np.int64)
    out[: keep.shape[0]] = keep
    return out


def topm_threshold(scores: np.ndarray, M: int) -> float:
    """Score of the M-th entry of the order (the lowest selected score)."""
    n = scores.shape[0]
    return float(scores[_order(scores)[min(M, n) - 1]])


def borderline_mask(scores: np.ndarray, M: int, rel: float = 1e-4, floor: float = 1e-3) -> np.ndarray:
    """Tokens whose selection may legitimately differ between the fp64 oracle
    and an fp32 device: |I(s) - s_M| <= rel * max(|s_M|, floor * max_s I(s)).
    Empty when n <= M (everything is selected)."""
    n = scores.shape[0]
    if n <= M:
        return np.zeros(n, dtype=bool)
    sM = topm_threshold(scores, M)
    tol = rel * max(abs(sM), floor * float(np.max(np.abs(scores))))
    return np.abs(scores - sM) <= tol


# --------------------------------------------------------------------------
# step 3: sparse softmax attention over the selected rows     [abs]
# --------------------------------------------------------------------------
def sparse_attention(q_h: np.ndarray, K_sel: np.ndarray, V_sel: np.ndarray) -> np.ndarray:
    """softmax_s(q . k_s / sqrt(d)) weighted sum of v_s over the given rows.

    q_h [d]; K_sel, V_sel [m, d] with m >= 1."""
    d = q_h.shape[0]
    logits = (K_sel @ q_h) / np.sqrt(d)
    p = np.exp(logits - np.max(logits))
    p = p / np.sum(p)
    return p @ V_sel


# --------------------------------------------------------------------------
# step 4: linear attention, phi = identity     [meth]
# --------------------------------------------------------------------------
def linear_update(S_h: np.ndarray, k_t: np.ndarray, v_t: np.ndarray) -> np.ndarray:
    """S <- S + k^T v  (S[i, j] += k[i] * v[j]); returns the new state."""
    return S_h + np.outer(k_t, v_t)


def linear_readout(q_h: np.ndarray, S_h: np.ndarray) -> np.ndarray:
    """o_lin[j] = sum_i q[i] * S[i, j]."""
    return q_h @ S_h


# --------------------------------------------------------------------------
# step 5: gate                                   [abs], [meth]
# --------------------------------------------------------------------------
def gate_fuse(lam: float, o_sp: np.ndarray, o_lin: np.ndarray) -> np.ndarray:
    """g = 1 / (1 + exp(-lam)); o = g * o_sp + (1 - g) * o_lin."""
    with np.errstate(over="ignore"):
        g = 1.0 / (1.0 + np.exp(-float(lam)))
    return g * o_sp + (1.0 - g) * o_lin


# --------------------------------------------------------------------------
# whole layer: one decode step
# --------------------------------------------------------------------------
def decode_step(q, k, v, qidx, kidx, w, lam, k_cache, v_cache, kidx_cache, S, pos, M,
                sel_override=None, shared_set=False, k_lin=None, v_lin=None):
    """One decode step for a batch.

    q [B,Hq,d]; k, v [B,Hkv,d]; qidx [B,HI,dI]; kidx [B,P,dI]; w [B,HI];
    lam [B,Hq]; caches [B,Hkv|P,>=pos[b],*] hold rows 0..pos[b]-1; S [B,Hq,d,d];
    pos [B] = position t of the new token.  P (indexer key planes) is Hkv by
    default, HI for one indexer key per indexer head, and 1 (or HI) with
    shared_set.
    sel_override: optional [B,Gs,M] index sets to use for the sparse branch
    instead of the oracle's own (the "conditional oracle").
    shared_set: one top-M set for every KV head, scored over all HI indexer
    heads (Gs = 1 selection group instead of Gs = Hkv).
    k_lin, v_lin: optional [B,Hq,d] keys / values of the linear branch, one
    per query head; by default the branch uses the attention's k, v of the
    head's KV group.

    Returns dict: out [B,Hq,d], idx [B,Gs,M], S [B,Hq,d,d],
    scores list (per b) of [Gs, t+1] arrays, o_sp, o_lin [B,Hq,d].
    """
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    Gs = 1 if shared_set else Hkv
    out = np.zeros((B, Hq, d))
    o_sp_all = np.zeros((B, Hq, d))
    o_lin_all = np.zeros((B, Hq, d))
    idx = np.full((B, Gs, M), -1, dtype=np.int64)
    S_new = np.array(S, dtype=np.float64, copy=True)
    scores_all = []
    for b in range(B):
        t = int(pos[b])
        # candidate keys 0..t: cached rows then the new token
        K = np.concatenate([k_cache[b, :, :t, :], k[b][:, None, :]], axis=1)          # [Hkv, t+1, d]
        V = np.concatenate([v_cache[b, :, :t, :], v[b][:, None, :]], axis=1)
        KI = np.concatenate([kidx_cache[b, :, :t, :], kidx[b][:, None, :]], axis=1)   # [P, t+1, dI]
        sc = indexer_scores(qidx[b], w[b], KI, groups=Gs)
        scores_all.append(sc)
        for gs in range(Gs):
            idx[b, gs] = topm_select(sc[gs], M)
        use = idx[b] if sel_override is None else np.asarray(sel_override[b])
        for h in range(Hq):
            g = h // G
            gs = 0 if shared_set else g
            sel = use[gs][use[gs] >= 0]
            o_sp = sparse_attention(q[b, h], K[g, sel], V[g, sel])
            kl_h = k[b, g] if k_lin is None else k_lin[b, h]
            vl_h = v[b, g] if v_lin is None else v_lin[b, h]
            S_new[b, h] = linear_update(S_new[b, h], kl_h, vl_h)
            o_lin = linear_readout(q[b, h], S_new[b, h])
            o_sp_all[b, h] = o_sp
            o_lin_all[b, h] = o_lin
            out[b, h] = gate_fuse(lam[b, h], o_sp, o_lin)
    return dict(out=out, idx=idx, S=S_new, scores=scores_all, o_sp=o_sp_all, o_lin=o_lin_all)


# --------------------------------------------------------------------------
# whole layer: causal prefill of T tokens
# --------------------------------------------------------------------------
def prefill(q, k, v, qidx, kidx, w, lam, S0, M, rows=None, sel_override=None, shared_set=False,
            k_lin=None, v_lin=None):
    """Causal prefill of T tokens starting from an empty cache.

    q [B,T,Hq,d]; k, v [B,T,Hkv,d]; qidx [B,T,HI,dI]; kidx [B,T,P,dI]
    (P as in decode_step); w [B,T,HI]; lam [B,T,Hq]; S0 [B,Hq,d,d].
    rows: optional iterable of token indices t whose outputs are wanted (the
    state always runs over all T tokens); default all.
    sel_override: optional callable (b, t) -> [Gs, M] index sets for the
    sparse branch (the "conditional oracle"), or None.
    shared_set, k_lin, v_lin ([B,T,Hq,d]): the variants of decode_step.

    Returns dict: out [B,T,Hq,d] (rows not requested stay 0), idx [B,T,Gs,M]
    (-1 for rows not requested), S [B,Hq,d,d] = state after token T-1,
    scores {(b, t): [Gs, t+1]} for the requested rows.
    """
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    Gs = 1 if shared_set else Hkv
    want = np.zeros(T, dtype=bool)
    if rows is None:
        want[:] = True
    else:
        want[np.asarray(list(rows), dtype=np.int64)] = True
    out = np.zeros((B, T, Hq, d))
    idx = np.full((B, T, Gs, M), -1, dtype=np.int64)
    S = np.array(S0, dtype=np.float64, copy=True)
    scores = {}
    for b in range(B):
        Kb = np.transpose(k[b], (1, 0, 2))        # [Hkv, T, d]
        Vb = np.transpose(v[b], (1, 0, 2))
        KIb = np.transpose(kidx[b], (1, 0, 2))    # [P, T, dI]
        for t in range(T):
            for h in range(Hq):
                kl_h = k[b, t, h // G] if k_lin is None else k_lin[b, t, h]
                vl_h = v[b, t, h // G] if v_lin is None else v_lin[b, t, h]
                S[b, h] = linear_update(S[b, h], kl_h, vl_h)
            if not want[t]:
                continue
            sc = indexer_scores(qidx[b, t], w[b, t], KIb[:, : t + 1, :], groups=Gs)
            scores[(b, t)] = sc
            for gs in range(Gs):
                idx[b, t, gs] = topm_select(sc[gs], M)
            use = idx[b, t] if sel_override is None else np.asarray(sel_override(b, t))
            for h in range(Hq):
                g = h // G
                gs = 0 if shared_set else g
                sel = use[gs][use[gs] >= 0]
                o_sp = sparse_attention(q[b, t, h], Kb[g, sel], Vb[g, sel])
                o_lin = linear_readout(q[b, t, h], S[b, h])
                out[b, t, h] = gate_fuse(lam[b, t, h], o_sp, o_lin)
    return dict(out=out, idx=idx, S=S, scores=scores)


# --------------------------------------------------------------------------
# Stage-2 indexer objective (forward): per-head KL      [abs]
# --------------------------------------------------------------------------
def indexer_kl(q, k, qidx, kidx, w, rows=None):
    """Per-head KL divergence between the frozen attention of each query
    head and the indexer's distribution over the causal prefix (arxivdaily.com
    English abstract: in Stage 2 the Indexer is trained with a per-head KL
    divergence that aligns its selection with the teacher's attention
    pattern).  Reading fixed here: for token t and query head h of KV head
    g = h // G,
        p_t,h(s) = softmax_{s <= t}(q[t,h] . k[s,g] / sqrt(d))      (teacher)
        r_t,g(s) = softmax_{s <= t}(I_g(t, s))                      (indexer)
        KL[t, h] = sum_s p_t,h(s) * (log p_t,h(s) - log r_t,g(s)).
    Tokens t = 0..T-1 of a sequence that starts at position 0.

    q [B,T,Hq,d]; k [B,T,Hkv,d]; qidx [B,T,HI,dI]; kidx [B,T,Hkv,dI]; w [B,T,HI].
    rows: optional token indices to evaluate (default all).
    Returns kl [B, T, Hq] (rows not requested stay 0).

    Parity: pinned by KL = 0 at t = 0, KL(p || uniform) = log(t+1) - H(p)
    when w = 0, and scipy's rel_entr on small inputs."""
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    kl = np.zeros((B, T, Hq))
    rows = range(T) if rows is None else rows
    for b in range(B):
        KIb = np.transpose(kidx[b], (1, 0, 2))                  # [Hkv, T, dI]
        for t in rows:
            sc = indexer_scores(qidx[b, t], w[b, t], KIb[:, : t + 1, :])   # [Hkv, t+1]
            for h in range(Hq):
                g = h // G
                a = (k[b, : t + 1, g, :] @ q[b, t, h]) / np.sqrt(d)
                pa = np.exp(a - a.max())
                pa /= pa.sum()
                c = sc[g]
                lr = c - c.max() - np.log(np.exp(c - c.max()).sum())     # log r
                la = np.log(np.maximum(pa, 1e-300))
                kl[b, t, h] = float(np.sum(pa * (la - lr)))
    return kl


# --------------------------------------------------------------------------
# projection front-end and output projection      [abs], [meth]
# --------------------------------------------------------------------------
# The abstract and the method details name the inputs of the layer -- the
# attention's q, k, v, the indexer's small query / key projections, the
# indexer head weights and the gate -- as projections of the hidden state,
# and the layer's output goes back to the hidden size.  The pages give no
# weights and no fused form; this library reads the front-end as ONE linear
# map of the hidden state whose output columns are, in this order,
#   q [Hq*d] | k [Hkv*d] | v [Hkv*d] | qidx [HI*dI] | kidx [P*dI] | w [HI] | lam [Hq]
# (P = Hkv indexer-key planes by default), and the output projection as the
# linear map o [Hq*d] -> y [Hm].  Weights are stored out-features x
# in-features (row n of W holds the weights of output column n).
PROJ_FIELDS = ("q", "k", "v", "qidx", "kidx", "w", "lam")


def proj_widths(Hq, Hkv, d, HI, dI, P=None):
    """Column count of every front-end field, in PROJ_FIELDS order."""
    P = Hkv if P is None else P
    return (Hq * d, Hkv * d, Hkv * d, HI * dI, P * dI, HI, Hq)


def project_in(x, W_in, Hq, Hkv, d, HI, dI, P=None):
    """Front-end: z = x W_in^T, split into the fields of the layer.

    x [..., Hm]; W_in [N_in, Hm] with N_in = sum(proj_widths(...)).
    Returns dict q [..., Hq, d], k, v [..., Hkv, d], qidx [..., HI, dI],
    kidx [..., P, dI], w [..., HI], lam [..., Hq].

    Parity: pinned by a brute-force triple loop on tiny inputs and by one-hot
    weight rows that route a chosen hidden coordinate into every field."""
    widths = proj_widths(Hq, Hkv, d, HI, dI, P)
    assert W_in.shape[0] == sum(widths), "W_in rows must equal the total field width"
    z = x @ W_in.T
    out, c = {}, 0
    shapes = {"q": (Hq, d), "k": (Hkv, d), "v": (Hkv, d), "qidx": (HI, dI),
              "kidx": (Hkv if P is None else P, dI), "w": (HI,), "lam": (Hq,)}
    for name, wd in zip(PROJ_FIELDS, widths):
        out[name] = z[..., c:c + wd].reshape(z.shape[:-1] + shapes[name])
        c += wd
    return out


def project_out(o, W_o):
    """Output projection y = o W_o^T.  o [..., Hq, d]; W_o [Hm, Hq*d].

    Parity: pinned by the brute-force loop and by W_o = identity (Hm = Hq*d)."""
    flat = o.reshape(o.shape[:-2] + (o.shape[-2] * o.shape[-1],))
    return flat @ W_o.T
