"""Plain fp64 CPU oracle of the MC-Sparse (Meta-Cached Sparse Attention) hot path.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The library's product
path never calls it, and this module imports nothing from the library: the two
share no code.  Inputs are bf16 bit patterns widened exactly to float64.

Sources (web pages describing the method; cited by title and section):

* [abstract] aiqbench.com, "MC-Sparse: Deconstructing and Closing the Dense-
  Sparse Attention Gap in Diffusion Transformers", the arXiv abstract.
* [p1-mcs] cnshai.top, "output-aware sparse attention / KV cache" post,
  section "MC-Sparse: three failure modes, one fix".
* [p1-trips] same post, section "What Trips People Up".
* [p4-design] cctest.ai, "MC-Sparse Narrows the Dense-Sparse Attention Gap in
  Diffusion Transformers", the list of three design choices.

What the pages fix: KV tokens are selected individually using exact attention
probabilities; similar queries are organised into tile-aligned groups; the
cached metadata are the query groups, the KV indices and the residual between
dense and sparse attention outputs, reused on later denoising steps
([abstract]; [p1-mcs]; [p4-design]).  Renormalising over the kept tokens is
not the dense result, which is why the residual is cached ([p1-trips]).

Readings taken where the pages are silent (each listed in the design notes):

* grouping: centre Q, take the eigenvector of the largest eigenvalue of the
  centred covariance (sign: its largest-magnitude component, lowest index on
  ties, is positive), project, stable ascending sort; groups are contiguous
  runs of G in that order, the last one partial.
* per-group score of key j: the sum over the group's queries of the exact
  softmax probability P_ij; keep the k' = min(k, N) largest, ties to the
  lower key index, stored ascending.
* sparse output: softmax renormalised over the kept keys; residual
  R_i = O_dense_i - O_sparse_i in the original token order; a reused step
  outputs O_sparse(current Q, K, V; cached groups and indices) + cached R.

Every function here is pinned by CPU tests against closed forms, brute force,
invariants or independent textbook routines; none is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "widen_bf16", "principal_direction", "projections", "group_queries",
    "group_rows", "scores", "row_stats", "probabilities", "group_prob_sums",
    "select_kv", "dense_rows", "dense_attention", "sparse_group",
    "sparse_attention", "residual_group", "plan_head", "reused_step_head",
    "rel_l2", "schedule_head",
    "select_blocks", "pooled_scores", "ungrouped_rows", "retained_mass",
    "round_bf16",
]


def widen_bf16(u16: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly."""
    u = np.asarray(u16, dtype=np.uint16)
    return (u.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def round_bf16(x) -> np.ndarray:
    """float32 values -> bf16 bit patterns (uint16), IEEE round to nearest,
    ties to even: of the two bf16 values bracketing x (x's float32 bits with
    the low 16 bits cleared, and the next bf16 away from zero) take the nearer;
    on a tie the one whose last mantissa bit is 0.  Magnitudes that round past
    the largest finite bf16 become infinity (the bracket above it counts as
    2^128, as in an unbounded exponent range).  NaN -> a quiet NaN.  (The
    storage format of the compact cached residual, a reading of this library,
    not of the pages.)"""
    with np.errstate(invalid="ignore"):
        return _round_bf16(np.ascontiguousarray(np.asarray(x, dtype=np.float32)))


def _round_bf16(x32: np.ndarray) -> np.ndarray:
    bits = x32.view(np.uint32)
    lo = (bits >> np.uint32(16)).astype(np.uint32)      # toward zero
    hi = lo + np.uint32(1)                               # away from zero
    mag = np.abs(x32.astype(np.float64))
    lo_v = np.abs(widen_bf16(lo.astype(np.uint16)))
    hi_exp_all_ones = (hi & np.uint32(0x7F80)) == np.uint32(0x7F80)
    hi_v = np.where(hi_exp_all_ones, 2.0 ** 128,
                    np.abs(widen_bf16((hi & np.uint32(0xFFFF)).astype(np.uint16))))
    d_lo, d_hi = mag - lo_v, hi_v - mag
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((lo & np.uint32(1)) == np.uint32(1)))
    exact = d_lo == 0.0
    out = np.where(take_hi & ~exact, hi, lo).astype(np.uint32)
    inf_or_nan = (bits & np.uint32(0x7F800000)) == np.uint32(0x7F800000)
    out = np.where(inf_or_nan, lo, out)                  # infinities are exact
    nan = np.isnan(x32)
    out = np.where(nan, np.uint32(0x7FC0), out)
    return (out & np.uint32(0xFFFF)).astype(np.uint16)


def _as_f64(x) -> np.ndarray:
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return widen_bf16(x)
    return x.astype(np.float64, copy=False)


# ---------------------------------------------------------------------------
# a1. Tile-aligned grouping of similar queries  ([abstract]; [p4-design]
#     "Hardware-aware query organization")
# ---------------------------------------------------------------------------

def principal_direction(Q):
    """Centre, covariance, top eigenpair of one head's queries.

    Returns (mu [d], C [d,d], v [d], eigenvalues ascending [d]).  v is the unit
    eigenvector of the largest eigenvalue, its sign fixed so that the first
    component of largest magnitude is positive.
    """
    Q = _as_f64(Q)
    n = Q.shape[0]
    mu = Q.mean(axis=0)
    X = Q - mu
    C = (X.T @ X) / n
    lam, U = np.linalg.eigh(C)
    v = U[:, -1].copy()
    i = int(np.argmax(np.abs(v)))
    if v[i] < 0:
        v = -v
    return mu, C, v, lam


def projections(Q, mu, v) -> np.ndarray:
    """p_n = (Q_n - mu) . v, each row's dot product summed on its own, so that
    equal query rows get equal projections and the stable sort keeps them in
    token order (a matrix-vector product may round equal rows differently,
    depending on where they fall in its row blocks and threads)."""
    return ((_as_f64(Q) - mu) * v).sum(axis=1)


def group_queries(Q) -> np.ndarray:
    """Query order perm (int64 [N]): stable ascending sort of the projections
    on the first principal direction.  Group g is perm[g*G : (g+1)*G]."""
    mu, _, v, _ = principal_direction(Q)
    p = projections(Q, mu, v)
    return np.argsort(p, kind="stable")


def group_rows(perm: np.ndarray, G: int, g: int) -> np.ndarray:
    return np.asarray(perm)[g * G:(g + 1) * G]


# ---------------------------------------------------------------------------
# a2. Exact attention probabilities  ([abstract] "KV indices selected using
#     exact attention probabilities"; [p4-design] "Individual KV selection")
# ---------------------------------------------------------------------------

def scores(Qrows, K, scale: float) -> np.ndarray:
    """s_ij = scale * Q_i . K_j"""
    return scale * (_as_f64(Qrows) @ _as_f64(K).T)


def row_stats(Qrows, K, scale: float):
    """m_i = max_j s_ij, l_i = sum_j exp(s_ij - m_i) over all N keys."""
    S = scores(Qrows, K, scale)
    m = S.max(axis=1)
    l = np.exp(S - m[:, None]).sum(axis=1)
    return m, l


def probabilities(Qrows, K, scale: float) -> np.ndarray:
    """P_ij = exp(s_ij - m_i) / l_i, the dense softmax rows."""
    S = scores(Qrows, K, scale)
    E = np.exp(S - S.max(axis=1, keepdims=True))
    return E / E.sum(axis=1, keepdims=True)


# ---------------------------------------------------------------------------
# a3 / a4. Per-group selection of individual KV tokens
# ---------------------------------------------------------------------------

def group_prob_sums(Q, K, scale: float, perm, G: int, groups=None) -> np.ndarray:
    """c[g, j] = sum over queries i of group g of P_ij.  [len(groups), N]"""
    Q = _as_f64(Q)
    K = _as_f64(K)
    n = Q.shape[0]
    ng = -(-n // G)
    groups = range(ng) if groups is None else groups
    out = np.empty((len(groups), K.shape[0]))
    for r, g in enumerate(groups):
        rows = group_rows(perm, G, g)
        out[r] = probabilities(Q[rows], K, scale).sum(axis=0)
    return out


def select_kv(c: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k' = min(k, N) largest entries of one group's score row,
    ties resolved towards the lower key index, returned ascending."""
    c = np.asarray(c, dtype=np.float64)
    n = c.shape[0]
    kk = min(int(k), n)
    order = np.lexsort((np.arange(n), -c))       # primary: -c, secondary: index
    return np.sort(order[:kk])


# ---------------------------------------------------------------------------
# a5 / a6 / a7. Dense output, renormalised sparse output, residual
#     ([abstract] "residuals between dense and sparse attention outputs";
#      [p1-trips] renormalising over the survivors is not a correction)
# ---------------------------------------------------------------------------

def dense_rows(Qrows, K, V, scale: float) -> np.ndarray:
    """O_i = sum_j P_ij V_j for the given query rows."""
    return probabilities(Qrows, K, scale) @ _as_f64(V)


def dense_attention(Q, K, V, scale: float, block: int = 0) -> np.ndarray:
    """Dense softmax(scale Q K^T) V of one head, query rows in blocks."""
    Q = _as_f64(Q)
    K = _as_f64(K)
    V = _as_f64(V)
    n = Q.shape[0]
    if block <= 0:
        block = max(16, min(1024, (1 << 26) // max(1, K.shape[0])))
    out = np.empty((n, V.shape[1]))
    for s in range(0, n, block):
        out[s:s + block] = dense_rows(Q[s:s + block], K, V, scale)
    return out


def sparse_group(Qrows, K, V, scale: float, idx) -> np.ndarray:
    """O_sp_i = sum_{j in S} exp(s_ij) V_j / sum_{j in S} exp(s_ij), softmax
    renormalised over the kept keys S only."""
    idx = np.asarray(idx)
    Ks = _as_f64(K)[idx]
    Vs = _as_f64(V)[idx]
    S = scores(Qrows, Ks, scale)
    E = np.exp(S - S.max(axis=1, keepdims=True))
    return (E / E.sum(axis=1, keepdims=True)) @ Vs


def sparse_attention(Q, K, V, scale: float, perm, kv_idx, G: int, groups=None):
    """Renormalised sparse output in original token order.  With `groups`
    given, returns (rows, O_sp[rows]) for those groups only."""
    Q = _as_f64(Q)
    n, d = Q.shape[0], _as_f64(V).shape[1]
    ng = -(-n // G)
    sel = range(ng) if groups is None else groups
    if groups is None:
        out = np.empty((n, d))
        for g in sel:
            rows = group_rows(perm, G, g)
            out[rows] = sparse_group(Q[rows], K, V, scale, kv_idx[g])
        return out
    rows_all, vals = [], []
    for g in sel:
        rows = group_rows(perm, G, g)
        rows_all.append(rows)
        vals.append(sparse_group(Q[rows], K, V, scale, kv_idx[g]))
    return np.concatenate(rows_all), np.concatenate(vals)


def residual_group(Qrows, K, V, scale: float, idx):
    """Residual of one group's rows, computed two ways.

    R = O_dense - O_sp (the definition), and R_alt = U - (1 - alpha) O_sp with
    U_i = sum_{j not in S} P_ij V_j and alpha_i = sum_{j in S} P_ij (the mass
    the kept keys hold under the dense softmax).  Returns (R, R_alt, alpha).
    """
    P = probabilities(Qrows, K, scale)
    Vf = _as_f64(V)
    O_dense = P @ Vf
    O_sp = sparse_group(Qrows, K, V, scale, idx)
    mask = np.zeros(P.shape[1], dtype=bool)
    mask[np.asarray(idx)] = True
    alpha = P[:, mask].sum(axis=1)
    U = P[:, ~mask] @ Vf[~mask]
    R = O_dense - O_sp
    R_alt = U - (1.0 - alpha)[:, None] * O_sp
    return R, R_alt, alpha


def plan_head(Q, K, V, G: int, k: int, scale: float):
    """The metadata pass of one head.

    Returns dict(perm int64 [N], kv_idx int64 [n_groups, k'], residual
    float64 [N, d] in original token order, O_dense float64 [N, d]).
    """
    Q = _as_f64(Q)
    K = _as_f64(K)
    V = _as_f64(V)
    n = Q.shape[0]
    d = V.shape[1]
    ng = -(-n // G)
    kk = min(int(k), n)
    perm = group_queries(Q)
    kv_idx = np.empty((ng, kk), dtype=np.int64)
    residual = np.empty((n, d))
    O_dense = np.empty((n, d))
    Vf = V
    for g in range(ng):
        rows = group_rows(perm, G, g)
        P = probabilities(Q[rows], K, scale)
        idx = select_kv(P.sum(axis=0), kk)
        kv_idx[g] = idx
        Od = P @ Vf
        Osp = sparse_group(Q[rows], K, V, scale, idx)
        O_dense[rows] = Od
        residual[rows] = Od - Osp
    return {"perm": perm, "kv_idx": kv_idx, "residual": residual, "O_dense": O_dense}


def reused_step_head(Q, K, V, scale: float, perm, kv_idx, residual, G: int, groups=None):
    """Reused denoising step: O_i = O_sp_i(current Q, K, V; cached groups and
    indices) + cached R_i.  With `groups`, returns (rows, O[rows])."""
    residual = np.asarray(residual, dtype=np.float64)
    if groups is None:
        return sparse_attention(Q, K, V, scale, perm, kv_idx, G) + residual
    rows, osp = sparse_attention(Q, K, V, scale, perm, kv_idx, G, groups=groups)
    return rows, osp + residual[rows]


# ---------------------------------------------------------------------------
# A denoising loop: plan on some steps, reuse the metadata on the others
# ---------------------------------------------------------------------------

def rel_l2(x, ref) -> float:
    """||x - ref|| / ||ref|| (Frobenius), in fp64."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / den) if den > 0 else float(np.linalg.norm(x))


def schedule_head(steps, plan_steps, G: int, k: int, scale: float):
    """One head through a denoising loop.

    ``steps`` lists the (Q, K, V) of denoising steps 1, 2, ...; ``plan_steps``
    holds the 1-based steps that compute fresh metadata (the first step always
    does, as nothing is cached before it).  The metadata -- query groups, KV
    indices and residual -- are computed once and reused on the following
    steps ([abstract]; [p1-mcs]): a plan step outputs the dense attention of
    its own inputs, a reused step outputs O_sparse(current Q, K, V; cached
    groups and indices) + cached R.

    Returns one dict per step: kind ("plan" or "reused"), the output O, the
    dense attention of that step's inputs, and the fidelity to it with the
    residual (rel_l2) and without it (rel_l2_no_residual, O - R).
    """
    plan_steps = set(int(t) for t in plan_steps)
    out = []
    meta = None
    for t, (Q, K, V) in enumerate(steps, start=1):
        if meta is None or t in plan_steps:
            meta = plan_head(Q, K, V, G, k, scale)
            kind, O = "plan", meta["O_dense"]
            Od = O
        else:
            kind = "reused"
            O = reused_step_head(Q, K, V, scale, meta["perm"], meta["kv_idx"], meta["residual"], G)
            Od = dense_attention(Q, K, V, scale)
        out.append({"step": t, "kind": kind, "O": O, "O_dense": Od,
                    "rel_l2": rel_l2(O, Od), "rel_l2_no_residual": rel_l2(O - meta["residual"], Od)})
    return out



# ---------------------------------------------------------------------------
# Synthetic ablations of the three failure modes the method addresses
#   ([abstract] "controlled oracle comparisons": the dense-sparse gap comes
#    from constraints imposed by token grouping, from inaccurate interaction
#    selection, and from the attention contributions lost; [p1-mcs] the three
#    failure modes and the one fix).  Each function below is the counterpart
#    of one MC-Sparse choice with that choice taken away.
# ---------------------------------------------------------------------------

def select_blocks(c: np.ndarray, k_blocks: int, block: int) -> np.ndarray:
    """Block-granular selection instead of individual tokens: the keys are cut
    into aligned blocks of `block` keys (a ragged last block is not a
    candidate), a block's score is the sum of its keys' scores, the
    k_blocks' = min(k_blocks, full blocks) highest blocks are kept (ties to the
    lower block index), and their keys are returned ascending."""
    c = np.asarray(c, dtype=np.float64)
    nb = c.shape[0] // block
    bs = c[:nb * block].reshape(nb, block).sum(axis=1)
    kb = min(int(k_blocks), nb)
    blocks = np.sort(np.lexsort((np.arange(nb), -bs))[:kb])
    return (blocks[:, None] * block + np.arange(block)[None, :]).reshape(-1)


def pooled_scores(Q, K, scale: float, perm, G: int, groups=None) -> np.ndarray:
    """A pooled, heuristic group score instead of exact summed probabilities:
    the group's queries are averaged into one query q_g and key j scores
    softmax_j(scale q_g . K_j), the probability the pooled query gives it.
    [len(groups), N]"""
    Q = _as_f64(Q)
    n = Q.shape[0]
    ng = -(-n // G)
    groups = range(ng) if groups is None else groups
    out = np.empty((len(groups), _as_f64(K).shape[0]))
    for r, g in enumerate(groups):
        qbar = Q[group_rows(perm, G, g)].mean(axis=0, keepdims=True)
        out[r] = probabilities(qbar, K, scale)[0]
    return out


def ungrouped_rows(Qrows, K, V, scale: float, k: int) -> np.ndarray:
    """No grouping constraint: every query keeps its own k' = min(k, N) largest
    exact probabilities (ties to the lower key index) and attends to them
    alone, renormalised.  [rows, d]"""
    Qrows = _as_f64(Qrows)
    P = probabilities(Qrows, K, scale)
    out = np.empty((Qrows.shape[0], _as_f64(V).shape[1]))
    for r in range(Qrows.shape[0]):
        out[r] = sparse_group(Qrows[r:r + 1], K, V, scale, select_kv(P[r], k))[0]
    return out


def retained_mass(c_row: np.ndarray, idx, size: int) -> float:
    """alpha_g: the share of group g's dense attention mass its kept keys hold,
    sum_{j in S_g} c_gj / |g| (c the group's summed exact probabilities)."""
    return float(np.asarray(c_row, dtype=np.float64)[np.asarray(idx)].sum() / size)
