"""Plain CPU oracle for one content-routed block-sparse attention (SSA) forward.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The product path (the CUDA library and its Python binding) never
imports, links or runs it, and this module imports nothing from the product.

Everything is computed in float64 with NumPy, step by step in the order the
method is stated, with no blocking or fusion:

  1. per-block key summaries: mean mu_c and (population) covariance Sigma_c,
     full or diagonal                       [Subquadratic Sparse Attention
     (SSA), opening section, step (i) "per-block summary statistics"]
  2. the second-cumulant routing score
         r_c(q) = <q, mu_c> + (beta/2) q^T Sigma_c q
     ("the block mean plus the variance of the logit across the block")
                                            [same page, "The idea in one
                                             screen", routing-score equation]
  3. a fixed budget of top-k blocks per query [same page, opening section,
     "fixed budget kappa << n"]
  4. union with a causal local window       [same page, opening section, (ii)]
  5. exact softmax attention over the selected keys
                                            [same page, opening section, (iii)]
  plus the closed-form recovery weight  w* = sigmoid(beta*Delta - log mu)
                                            [same page, "The idea in one
                                             screen", recovery-law equation]

Readings of points the pages leave open (each is listed with its reason in
the repository's design notes):
  * variance normaliser: population (1/B), which makes r_c an exact identity
    with the mean and variance of the block's logits;
  * routing uses raw q and raw keys; the attention scale is applied only
    inside attention;
  * a block is a routing candidate for the query at key position ``pos`` only
    when it is fully visible: (c+1)*B - 1 <= pos;
  * the window is the W keys pos-W+1 .. pos (the query's own key included);
  * the attended key set is the set union of the selected blocks' keys and
    the window keys (each key counted once);
  * fewer than k eligible blocks: take all of them, pad with -1;
  * ties: higher score first, then lower block index;
  * grouped-query attention: one selection per (token, kv-head), ranked by
    the sum over the group's query heads of r_c(q_h);
  * bf16 problems route on bf16 features and bf16 summaries whose rounding
    is part of the definition (``route_features`` / ``stored_summaries``);
  * the cascade's outlier channel (named on the same page, artifact list,
    without a rule): each block gets one more summary row, its key of
    largest 2-norm with a zero covariance, so the row scores that key's
    exact group logit; a block scores the larger of its two rows
    (``outlier_keys`` / ``with_outlier_rows``).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, brute force, invariants and hand-computed golden cases).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

F32 = "f32"
BF16 = "bf16"
DIAG = "diag"
FULL = "full"


@dataclass
class Problem:
    """Shape and hyper-parameters of one SSA forward (mirrors the C struct)."""
    batch: int
    n_q: int
    n_kv: int
    h_q: int
    h_kv: int
    d: int
    block: int
    topk: int
    window: int
    q_offset: int = 0
    beta: float = 2.0
    scale: float = field(default=float("nan"))
    dtype: str = BF16
    sigma: str = DIAG
    subblocks: int = 1          # sub-block summaries per block (max-pooled routing)
    outlier: bool = False       # one more summary row per block: its largest-norm key

    def __post_init__(self):
        if not math.isfinite(self.scale):
            self.scale = 1.0 / math.sqrt(self.d)

    @property
    def group(self) -> int:
        return self.h_q // self.h_kv

    @property
    def nb(self) -> int:
        return self.n_kv // self.block

    @property
    def unit(self) -> int:
        """Keys per summary: the block, or its sub-block when subblocks > 1."""
        return self.block // self.subblocks

    @property
    def rows_per_block(self) -> int:
        """Summary rows per block: the S sub-blocks, plus the outlier row."""
        return self.subblocks + (1 if self.outlier else 0)


# ---------------------------------------------------------------- rounding

def round_f32(x) -> np.ndarray:
    """Round to the nearest float32 (ties to even), returned as float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_bf16(x) -> np.ndarray:
    """Round float32 values to bfloat16, nearest with ties to even.

    bfloat16 keeps the top 16 bits of an IEEE float32.  Rounding adds half an
    ulp of the kept part (0x7FFF) plus the kept part's lowest bit (so that an
    exact half rounds to the even neighbour), then truncates.  Input is first
    rounded to float32 so the result is the float32 -> bfloat16 conversion.
    Returned as float64 (every bfloat16 value is exact there).
    """
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = a.view(np.uint32).astype(np.uint64)
    keep_lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + keep_lsb) >> np.uint64(16)) << np.uint64(16)
    out = (r & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)
    return out.astype(np.float64)


# ---------------------------------------------------------------- step 1

def block_summaries(K: np.ndarray, p: Problem):
    """Per-(batch, kv-head, block) key mean and population covariance.

    K: [batch, n_kv, h_kv, d].  Returns (mu, sig) in float64:
      mu  [batch, h_kv, nb, d]       mu_c = (1/B) sum_{j in c} k_j
      sig [batch, h_kv, nb, d]       diagonal: (1/B) sum_j (k_j - mu_c)_t^2
      sig [batch, h_kv, nb, d, d]    full:     (1/B) sum_j (k_j - mu_c)(k_j - mu_c)^T
    With p.subblocks = S > 1 the summaries are taken per sub-block of B/S
    consecutive keys instead (nb * S rows, sub-block s of block c at c*S + s).
    With p.outlier each block gets a second row, its largest-norm key with a
    zero covariance (row 2c+1; see with_outlier_rows).
    """
    b, n, h, d = K.shape
    B = p.unit
    nb = n // B
    Kb = np.asarray(K, dtype=np.float64).reshape(b, nb, B, h, d).transpose(0, 3, 1, 2, 4)
    mu = Kb.sum(axis=3) / B
    dev = Kb - mu[:, :, :, None, :]
    if p.sigma == FULL:
        sig = np.einsum("xhcjs,xhcjt->xhcst", dev, dev) / B
    else:
        sig = (dev * dev).sum(axis=3) / B
    if p.outlier:
        mu, sig = with_outlier_rows(K, mu, sig, p)
    return mu, sig


def outlier_keys(K: np.ndarray, p: Problem) -> np.ndarray:
    """The outlier channel's key of every block: the key of largest 2-norm
    (squared norms in float64; equal norms go to the earlier key).
    Returns [batch, h_kv, nb, d] float64."""
    b, n, h, d = K.shape
    nb = n // p.block
    Kb = np.asarray(K, dtype=np.float64).reshape(b, nb, p.block, h, d).transpose(0, 3, 1, 2, 4)
    norm2 = (Kb * Kb).sum(axis=-1)                       # [b, h, nb, B]
    j = np.argmax(norm2, axis=-1)                        # first of equal maxima
    return np.take_along_axis(Kb, j[..., None, None], axis=3)[:, :, :, 0, :]


def with_outlier_rows(K: np.ndarray, mu: np.ndarray, sig: np.ndarray, p: Problem):
    """Interleaves the outlier rows after each block's summary row: row 2c is
    block c's (mean, covariance), row 2c+1 its largest-norm key k*_c with a
    zero covariance, so that the row's score is the group logit of k*_c
    (sub-block summaries are not combined with the outlier row)."""
    if p.subblocks != 1:
        raise ValueError("the outlier row is defined for whole-block summaries")
    ko = outlier_keys(K, p)
    b, h, nb, d = mu.shape
    mu2 = np.empty((b, h, 2 * nb, d))
    mu2[:, :, 0::2], mu2[:, :, 1::2] = mu, ko
    sig2 = np.zeros((b, h, 2 * nb) + sig.shape[3:])
    sig2[:, :, 0::2] = sig
    return mu2, sig2


def stored_summaries(mu: np.ndarray, sig: np.ndarray, p: Problem):
    """The summary values the router reads.

    fp32 problems: mu and Sigma rounded to float32.  bf16 problems (diagonal
    only): the float32 values rounded once more to bfloat16, packed per block
    as the routing row [mu_c ; sigma_c^2] of length 2d.
    Returns (mu32, sig32, table) with table None for fp32 problems.
    """
    mu32 = round_f32(mu)
    sig32 = round_f32(sig)
    if p.dtype == F32:
        return mu32, sig32, None
    if p.sigma != DIAG:
        raise ValueError("bf16 routing is defined for diagonal Sigma only")
    table = np.concatenate([round_bf16(mu32), round_bf16(sig32)], axis=-1)
    return mu32, sig32, table


# ---------------------------------------------------------------- step 2

def route_features(Q: np.ndarray, p: Problem) -> np.ndarray:
    """bf16 routing features per (batch, kv-head, query row), length 2d.

    For the query heads h of kv-head g (in head order):
        qs = sum_h q_h            (float32 additions, head order)
        qq = sum_h q_h * q_h      (float32; each product of bf16 values is exact)
        f  = [bf16(qs), bf16(float32(beta/2) * qq)]
    so that f . [mu_c ; sigma_c^2] = sum_h r_c(q_h) up to the stated rounding.
    Q: [batch, n_q, h_q, d].  Returns [batch, h_kv, n_q, 2d] float64.
    """
    b, nq, hq, d = Q.shape
    G = p.group
    Qg = np.asarray(Q, dtype=np.float32).reshape(b, nq, p.h_kv, G, d)
    qs = np.zeros((b, nq, p.h_kv, d), dtype=np.float32)
    qq = np.zeros((b, nq, p.h_kv, d), dtype=np.float32)
    for h in range(G):
        qh = Qg[:, :, :, h, :]
        qs = (qs + qh).astype(np.float32)
        qq = (qq + qh * qh).astype(np.float32)
    half_beta = np.float32(np.float32(p.beta) * np.float32(0.5))
    f = np.concatenate([round_bf16(qs), round_bf16((half_beta * qq).astype(np.float32))], axis=-1)
    return f.transpose(0, 2, 1, 3)


def visible_blocks(pos: int, p: Problem) -> int:
    """Number of fully visible blocks for key position pos: (c+1)B-1 <= pos."""
    return max(0, min(p.nb, (pos + 1) // p.block))


# ---------------------------------------------------------------- step 2 (scores)

def pool_subblocks(scores: np.ndarray, p: Problem) -> np.ndarray:
    """Block scores from summary-row scores (last axis nb * R, R rows per
    block: the S sub-blocks and the outlier row): the maximum over each
    block's rows (identity for R = 1)."""
    S = p.rows_per_block
    if S == 1:
        return scores
    sh = scores.shape
    return scores.reshape(sh[:-1] + (sh[-1] // S, S)).max(axis=-1)


def route_scores_row(Q: np.ndarray, stored, p: Problem, bi: int, i: int, g: int) -> np.ndarray:
    """Routing scores of query row i (batch bi, kv-head g) for all visible blocks.

    bf16: s_c = f . [mu_c ; sigma_c^2] with the bf16 features and table.
    fp32: s_c = sum_h ( <q_h, mu_c> + (beta/2) q_h^T Sigma_c q_h ) with the
          float32 summaries (diagonal Sigma: q_h^T diag(sigma^2) q_h).
    With sub-block summaries each score is taken per sub-block and a block
    scores the largest of its sub-blocks' (group-summed) scores.
    """
    mu32, sig32, table = stored
    nv = visible_blocks(p.q_offset + i, p)
    nu = nv * p.rows_per_block                 # visible summary rows
    if p.dtype == BF16:
        f = route_features(Q[bi:bi + 1, i:i + 1], p)[0, g, 0]
        return pool_subblocks(table[bi, g, :nu] @ f, p)
    G = p.group
    q = np.asarray(Q[bi, i, g * G:(g + 1) * G], dtype=np.float64)  # [G, d]
    mu = mu32[bi, g, :nu]                                           # [nu, d]
    s = (q @ mu.T).sum(axis=0)
    if p.sigma == FULL:
        quad = np.einsum("hs,cst,ht->c", q, sig32[bi, g, :nu], q)
    else:
        quad = ((q * q) @ sig32[bi, g, :nu].T).sum(axis=0)
    return pool_subblocks(s + (p.beta / 2.0) * quad, p)


def route_scores(Q: np.ndarray, stored, p: Problem, bi: int, g: int) -> np.ndarray:
    """All rows of one (batch, kv-head): [n_q, nb] with -inf where not visible."""
    mu32, sig32, table = stored
    out = np.full((p.n_q, p.nb), -np.inf)
    if p.dtype == BF16:
        f = route_features(Q[bi:bi + 1], p)[0, g]          # [n_q, 2d]
        full = f @ table[bi, g].T                          # [n_q, nb]
    else:
        G = p.group
        q = np.asarray(Q[bi, :, g * G:(g + 1) * G], dtype=np.float64)  # [n_q, G, d]
        full = np.einsum("ihd,cd->ic", q, mu32[bi, g])
        if p.sigma == FULL:
            full = full + (p.beta / 2.0) * np.einsum("ihs,cst,iht->ic", q, sig32[bi, g], q)
        else:
            full = full + (p.beta / 2.0) * np.einsum("ihd,cd->ic", q * q, sig32[bi, g])
    full = pool_subblocks(full, p)
    for i in range(p.n_q):
        nv = visible_blocks(p.q_offset + i, p)
        out[i, :nv] = full[i, :nv]
    return out


def tempered_block_score(q: np.ndarray, Kc: np.ndarray, beta: float) -> float:
    """The tempered block score  T_beta = (1/beta) log( (1/B) sum_j exp(beta <q, k_j>) )
    over the B keys of one block (beta = 0: the mean logit).

    The routing score's family ["Subquadratic Sparse Attention (SSA)",
    artifact list: the temperature family interpolating centroid <->
    cumulant <-> exact-max]: T_beta is the block's log-mean-exp of the scaled
    logits; beta -> 0 gives the centroid score <q, mu_c>, its second-order
    expansion in beta is the cumulant score <q, mu_c> + (beta/2) q^T Sigma_c q,
    and beta -> infinity gives max_j <q, k_j>.  Needs every key of the block,
    so it is an analysis reference, not a summary-only router.
    """
    s = np.asarray(Kc, dtype=np.float64) @ np.asarray(q, dtype=np.float64)
    if beta == 0.0:
        return float(s.mean())
    m = s.max()
    return float(m + np.log(np.mean(np.exp(beta * (s - m)))) / beta)


# ---------------------------------------------------------------- step 3

def select_topk(scores: np.ndarray, k: int):
    """Top-k of one row of visible-block scores under (score desc, index asc).

    Returns (block_idx[k] ascending, padded with -1;  rel_gap) where rel_gap is
    (s_k - s_{k+1}) / |s_k| when more than k blocks are visible, else +inf.
    """
    nv = scores.shape[0]
    idx = np.arange(nv)
    order = np.lexsort((idx, -scores))           # primary: -score, then index
    take = min(k, nv)
    sel = np.sort(order[:take])
    out = np.full(k, -1, dtype=np.int64)
    out[:take] = sel
    if nv > k:
        sk, sk1 = scores[order[k - 1]], scores[order[k]]
        gap = (sk - sk1) / abs(sk) if sk != 0 else (np.inf if sk > sk1 else 0.0)
    else:
        gap = np.inf
    return out, gap


def route_topk(Q: np.ndarray, stored, p: Problem, rows=None):
    """block_idx [batch, n_q, h_kv, k] and relative k/k+1 gaps [batch, n_q, h_kv].

    rows: optional list of (batch, query row) pairs; other rows are left -2.
    """
    bidx = np.full((p.batch, p.n_q, p.h_kv, p.topk), -2, dtype=np.int64)
    gaps = np.full((p.batch, p.n_q, p.h_kv), np.nan)
    if rows is None:
        for bi in range(p.batch):
            for g in range(p.h_kv):
                S = route_scores(Q, stored, p, bi, g)
                for i in range(p.n_q):
                    nv = visible_blocks(p.q_offset + i, p)
                    bidx[bi, i, g], gaps[bi, i, g] = select_topk(S[i, :nv], p.topk)
    else:
        for bi, i in rows:
            for g in range(p.h_kv):
                s = route_scores_row(Q, stored, p, bi, i, g)
                bidx[bi, i, g], gaps[bi, i, g] = select_topk(s, p.topk)
    return bidx, gaps


def route_topk_unquantised(Q: np.ndarray, stored, p: Problem, rows=None):
    """The selection of a bf16 problem without its bf16 rounding of features
    and summaries, for information: the same cumulant scores from the float64
    query heads and the float32 summaries, i.e. exactly what the float32
    problem computes (``route_topk`` on a float32 copy of the problem)."""
    mu32, sig32, _table = stored
    q32 = Problem(**{**p.__dict__, "dtype": F32})
    return route_topk(Q, (mu32, sig32, None), q32, rows)


# ---------------------------------------------------------------- step 4

def key_set(pos: int, sel: np.ndarray, p: Problem) -> np.ndarray:
    """Sorted key indices attended by the query at position pos.

    Union of the selected blocks' keys and the window keys pos-W+1 .. pos.
    """
    blocks = [np.arange(c * p.block, (c + 1) * p.block) for c in sel if c >= 0]
    win = np.arange(max(0, pos - p.window + 1), pos + 1)
    return np.union1d(np.concatenate(blocks + [win]), np.array([], dtype=np.int64)).astype(np.int64)


# ---------------------------------------------------------------- step 5

def softmax_attend(q: np.ndarray, Ks: np.ndarray, Vs: np.ndarray, scale: float):
    """Exact softmax attention of query heads q [G, d] over keys Ks/Vs [m, d].

    Returns (o [G, d], lse [G]) with lse = log sum_j exp(scale * q.k_j).
    """
    logits = (np.asarray(q, np.float64) @ np.asarray(Ks, np.float64).T) * scale
    m = logits.max(axis=1, keepdims=True)
    w = np.exp(logits - m)
    l = w.sum(axis=1, keepdims=True)
    o = (w @ np.asarray(Vs, np.float64)) / l
    return o, (m + np.log(l))[:, 0]


def attention(Q, K, V, block_idx, p: Problem, rows=None):
    """Gathered exact attention for every (batch, query row) or for ``rows``.

    Returns O [batch, n_q, h_q, d] and lse [batch, n_q, h_q] (NaN where not
    computed).
    """
    O = np.full((p.batch, p.n_q, p.h_q, p.d), np.nan)
    L = np.full((p.batch, p.n_q, p.h_q), np.nan)
    if rows is None:
        rows = [(bi, i) for bi in range(p.batch) for i in range(p.n_q)]
    G = p.group
    for bi, i in rows:
        pos = p.q_offset + i
        for g in range(p.h_kv):
            S = key_set(pos, block_idx[bi, i, g], p)
            o, lse = softmax_attend(Q[bi, i, g * G:(g + 1) * G], K[bi, S, g], V[bi, S, g], p.scale)
            O[bi, i, g * G:(g + 1) * G] = o
            L[bi, i, g * G:(g + 1) * G] = lse
    return O, L


def dense_causal_attention(Q, K, V, p: Problem):
    """Dense causal softmax attention over all keys j <= pos (full matrices)."""
    b, nq, hq, d = Q.shape
    G = p.group
    O = np.zeros((b, nq, hq, d))
    L = np.zeros((b, nq, hq))
    pos = p.q_offset + np.arange(nq)
    mask = np.arange(p.n_kv)[None, :] <= pos[:, None]              # [nq, nkv]
    for bi in range(b):
        for h in range(hq):
            g = h // G
            logits = (np.asarray(Q[bi, :, h], np.float64) @ np.asarray(K[bi, :, g], np.float64).T) * p.scale
            logits = np.where(mask, logits, -np.inf)
            m = logits.max(axis=1, keepdims=True)
            w = np.exp(logits - m)
            l = w.sum(axis=1, keepdims=True)
            O[bi, :, h] = (w @ np.asarray(V[bi, :, g], np.float64)) / l
            L[bi, :, h] = (m + np.log(l))[:, 0]
    return O, L


# ---------------------------------------------------------------- whole layer

def forward(Q, K, V, p: Problem, rows=None):
    """The whole layer: summaries -> route -> top-k -> key set -> attention.

    Returns dict with O, lse, block_idx, gaps and the stored summaries.
    """
    mu, sig = block_summaries(K, p)
    stored = stored_summaries(mu, sig, p)
    bidx, gaps = route_topk(Q, stored, p, rows)
    O, L = attention(Q, K, V, bidx, p, rows)
    return {"O": O, "lse": L, "block_idx": bidx, "gaps": gaps,
            "mu": mu, "sig": sig, "stored": stored}


# ---------------------------------------------------------------- closed forms

def recovery_weight(beta: float, delta: float, mu: float) -> float:
    """w* = sigmoid(beta * Delta - log mu): softmax weight of one target whose
    logit margin over each of mu equal distractors is Delta (at inverse
    temperature beta)."""
    return 1.0 / (1.0 + math.exp(-(beta * delta - math.log(mu))))


# ---------------------------------------------------------------- hierarchical router

# The page "Subquadratic Sparse Attention (SSA)" names, without defining them,
# a tree router with a recursive radius (its artifact list, Barnes-Hut style),
# exact branch-and-bound selection under an admissible bound (same list) and
# per-query certificates with escalation (the "Certified Causal Cascade"
# entry).  The reading written out below:
#
#   * a node is M consecutive blocks (M = the fan-out); only complete nodes
#     exist, a trailing group of fewer than M blocks is no node;
#   * node summary, from the stored bf16 routing rows T_c = [mu_c ; s_c] of its
#     blocks: centre m_N = bf16(f32(mean_c mu_c)), variance cap
#     v_N = max_c s_c (per dimension), radius R_N = max_c ||mu_c - m_N||_2
#     (float64, rounded up to float32);
#   * admissible bound: for any block c of N and features f = [f_s ; f_q]
#     with f_q >= 0,  f . T_c <= f . [m_N ; v_N] + ||f_s|| R_N
#     (Cauchy-Schwarz on the mean part, the cap on the variance part);
#   * a query row ranks its complete visible nodes by w_N = f . [m_N ; v_N]
#     (higher first, then lower node index), expands the first p, scores
#     exactly every block of those nodes and every visible block outside a
#     complete visible node, and keeps the top-k of those scores;
#   * certificate: the row is certified when no complete visible node is left
#     unexpanded, or when its k-th kept score exceeds
#     w_(p+1) + ||f_s|| R* + margin, with R* the largest radius of the
#     (batch, kv-head) and margin = 2^-12 ||f|| T*, T* the largest 2-norm of
#     any of its block or node rows (room for float32 rounding of both
#     sides).  Every unexpanded block then scores below the k-th kept score,
#     so the kept set is the exact top-k of all visible blocks;
#   * escalation: an uncertified row is re-routed over all its visible blocks.
#
# Listed outlier blocks (optional, parameter lambda >= 1): block c of a
# complete node N is listed when the 2-norm of its variance half s_c exceeds
# lambda times the node's lower median of those norms (the (M/2)-th
# smallest).  The node's centre, cap and radius then come from its unlisted
# blocks only (the mean divides by their count; at least half of the blocks
# are unlisted), and a row scores exactly every listed block of its complete
# visible nodes beside the blocks of its expanded nodes and the tail.  The
# bound and the certificate are unchanged: they now cover the unlisted
# blocks, and every listed block is a candidate.  (A block whose variance
# stands far above its neighbours' -- a block holding one extreme key --
# would otherwise lift the node's cap in every dimension.)

HIER_MARGIN = 2.0 ** -12


def round_up_f32(x) -> np.ndarray:
    """The least float32 >= x (x finite, float64), returned as float64."""
    x = np.asarray(x, dtype=np.float64)
    r = x.astype(np.float32)
    low = r.astype(np.float64) < x
    r = np.where(low, np.nextafter(r, np.float32(np.inf)), r)
    return r.astype(np.float64)


def hier_listed_blocks(table: np.ndarray, fanout: int, factor: float) -> np.ndarray:
    """listed [batch, h_kv, nb] (bool): block c of complete node N is listed
    when ||s_c||_2 > factor * (the (M/2)-th smallest ||s||_2 of N's blocks),
    s_c the variance half of its stored row; blocks outside complete nodes
    are never listed."""
    b, h, nb, kf = table.shape
    d = kf // 2
    M = fanout
    nn = nb // M
    vn = np.sqrt((np.asarray(table, dtype=np.float64)[..., d:] ** 2).sum(axis=-1))   # [b, h, nb]
    listed = np.zeros((b, h, nb), dtype=bool)
    if nn:
        node_vn = vn[:, :, :nn * M].reshape(b, h, nn, M)
        lower_median = np.sort(node_vn, axis=3)[..., M // 2 - 1] if M > 1 else node_vn[..., 0]
        listed[:, :, :nn * M] = (node_vn > factor * lower_median[..., None]).reshape(b, h, nn * M)
    return listed


def hier_nodes(table: np.ndarray, fanout: int, listed=None):
    """Node summaries of a bf16 routing table [batch, h_kv, nb, 2d].

    Returns (node_table [batch, h_kv, nn, 2d] bf16 values, radius
    [batch, h_kv, nn], r_star [batch, h_kv], t_star [batch, h_kv]) with
    nn = nb // fanout; r_star / t_star are 0 when there are no nodes or rows.
    listed [batch, h_kv, nb] (optional): blocks left out of their node's
    centre, cap and radius.
    """
    b, h, nb, kf = table.shape
    d = kf // 2
    M = fanout
    nn = nb // M
    T = np.asarray(table, dtype=np.float64)
    nodes = T[:, :, :nn * M].reshape(b, h, nn, M, kf)
    keep = np.ones((b, h, nn, M), dtype=bool)
    if listed is not None:
        keep = ~np.asarray(listed, dtype=bool)[:, :, :nn * M].reshape(b, h, nn, M)
    count = keep.sum(axis=3)
    centre = round_bf16(round_f32((nodes[..., :d] * keep[..., None]).sum(axis=3) / np.maximum(count, 1)[..., None]))
    cap = np.where(keep[..., None], nodes[..., d:], -np.inf).max(axis=3) if nn else np.zeros((b, h, 0, d))
    dist = np.sqrt(((nodes[..., :d] - centre[:, :, :, None, :]) ** 2).sum(axis=-1))   # [b, h, nn, M]
    radius = round_up_f32(np.where(keep, dist, 0.0).max(axis=3)) if nn else np.zeros((b, h, 0))
    node_table = np.concatenate([centre, cap], axis=-1)
    r_star = radius.max(axis=2) if nn else np.zeros((b, h))
    row_norm = np.sqrt((T ** 2).sum(axis=-1))
    node_norm = np.sqrt((node_table ** 2).sum(axis=-1))
    t_star = np.zeros((b, h))
    if nb:
        t_star = row_norm.max(axis=2)
    if nn:
        t_star = np.maximum(t_star, node_norm.max(axis=2))
    return node_table, radius, round_up_f32(r_star), round_up_f32(t_star)


def hier_super_nodes(node_table: np.ndarray, radius: np.ndarray, t_star: np.ndarray, fanout: int):
    """The tree's second level over the node table [batch, h_kv, nn, 2d].

    Super-node S = nodes S*M .. S*M+M-1 (complete super-nodes only): centre
    bf16(f32(mean of the nodes' centres)), cap = per-dimension maximum of the
    nodes' caps, and the recursive radius max_N (||m_N - m_S|| + R_N) (float64,
    rounded up to float32): by the triangle inequality every block mean of
    S lies within it of m_S.  Returns (super_table [batch, h_kv, ns, 2d],
    super_radius [batch, h_kv, ns], r2_star [batch, h_kv] (0 without
    super-nodes), t_star raised to the super-node rows' largest 2-norm).
    """
    b, h, nn, kf = node_table.shape
    d = kf // 2
    M = fanout
    ns = nn // M
    N = np.asarray(node_table, dtype=np.float64)
    kids = N[:, :, :ns * M].reshape(b, h, ns, M, kf)
    centre = round_bf16(round_f32(kids[..., :d].sum(axis=3) / M))
    cap = kids[..., d:].max(axis=3) if ns else np.zeros((b, h, 0, d))
    kid_r = np.asarray(radius, dtype=np.float64)[:, :, :ns * M].reshape(b, h, ns, M)
    dist = np.sqrt(((kids[..., :d] - centre[:, :, :, None, :]) ** 2).sum(axis=-1))   # [b, h, ns, M]
    sradius = round_up_f32((dist + kid_r).max(axis=3)) if ns else np.zeros((b, h, 0))
    stable = np.concatenate([centre, cap], axis=-1)
    r2_star = round_up_f32(sradius.max(axis=2)) if ns else np.zeros((b, h))
    t2 = np.asarray(t_star, dtype=np.float64)
    if ns:
        t2 = np.maximum(t2, round_up_f32(np.sqrt((stable ** 2).sum(axis=-1)).max(axis=2)))
    return stable, sradius, r2_star, t2


def hier_route_row(f: np.ndarray, table_bg: np.ndarray, nodes_bg, pos: int, p: Problem, fanout: int,
                   probe: int, listed_bg=None):
    """One (query row, kv-head) through the hierarchical router.

    f: the row's features [2d]; table_bg [nb, 2d]; nodes_bg = (node_table
    [nn, 2d], radius [nn], r_star, t_star) of its (batch, kv-head);
    listed_bg [nb] (optional): listed blocks, candidates of every row that
    sees their node and no part of an expanded node's candidates.
    Returns (kept block_idx [k] ascending padded with -1, certified,
    info dict with the expanded nodes, the node gap and the kept-set gap).
    """
    node_table, _radius, r_star, t_star = nodes_bg
    d = p.d
    M = fanout
    nn = node_table.shape[0]
    nv = visible_blocks(pos, p)
    nvn = max(0, min(nn, (pos + 1) // (M * p.block)))
    w = node_table[:nvn] @ f
    order = np.lexsort((np.arange(nvn), -w))
    expanded = np.sort(order[:probe])
    cand = [np.arange(N * M, (N + 1) * M) for N in expanded] + [np.arange(nvn * M, nv)]
    cand = np.concatenate(cand).astype(np.int64)
    if listed_bg is not None:
        lst = np.asarray(listed_bg, dtype=bool)
        in_nodes = cand < nvn * M
        cand = np.concatenate([cand[~(in_nodes & lst[cand])], np.flatnonzero(lst[:nvn * M])]).astype(np.int64)
    s = table_bg[cand] @ f
    corder = np.lexsort((cand, -s))
    take = min(p.topk, cand.size)
    kept = np.full(p.topk, -1, dtype=np.int64)
    kept[:take] = np.sort(cand[corder[:take]])
    tau = s[corder[p.topk - 1]] if cand.size >= p.topk else -np.inf
    f_s_norm = math.sqrt(float(f[:d] @ f[:d]))
    margin = HIER_MARGIN * math.sqrt(float(f @ f)) * t_star
    if nvn <= probe:
        certified, w_next, node_gap = True, -np.inf, np.inf
    else:
        w_next = w[order[probe]]
        certified = bool(tau > w_next + f_s_norm * r_star + margin)
        node_gap = w[order[probe - 1]] - w_next
    kgap = (s[corder[p.topk - 1]] - s[corder[p.topk]]) if cand.size > p.topk else np.inf
    info = {"expanded": expanded, "tau": tau, "bound": w_next + f_s_norm * r_star + margin,
            "node_gap": node_gap, "kept_gap": kgap, "scale": math.sqrt(float(f @ f)) * t_star}
    return kept, certified, info


def hier_route_row2(f: np.ndarray, table_bg: np.ndarray, nodes_bg, supers_bg, pos: int, p: Problem,
                    fanout: int, probe: int):
    """One (query row, kv-head) through the two-level tree.

    supers_bg = (super_table [ns, 2d], super_radius [ns], r2_star, t_star)
    of its (batch, kv-head); nodes_bg as for hier_route_row (its t_star is
    replaced by the one covering the super-node rows).  The row ranks its
    complete visible super-nodes by w_S = f . [m_S ; v_S] and expands the best
    `probe`; their nodes and the complete visible nodes outside complete
    super-nodes are ranked by w_N, the best `probe` of them expanded; the
    blocks of those and the visible blocks outside complete nodes are scored
    exactly and their top-k kept.  Certified when neither level leaves an
    unexpanded entry whose bound (w + ||f_s|| R* + margin, R* the level's
    largest radius) reaches the k-th kept score.
    """
    node_table, _radius, r_star, _t1 = nodes_bg
    stable, _sradius, r2_star, t_star = supers_bg
    d = p.d
    M = fanout
    nn = node_table.shape[0]
    ns = stable.shape[0]
    nv = visible_blocks(pos, p)
    nvn = max(0, min(nn, (pos + 1) // (M * p.block)))
    nvs = max(0, min(ns, (pos + 1) // (M * M * p.block)))
    w2 = stable[:nvs] @ f
    order2 = np.lexsort((np.arange(nvs), -w2))
    sexp = np.sort(order2[:probe])
    ncand = np.concatenate([np.arange(S * M, (S + 1) * M) for S in sexp] +
                           [np.arange(nvs * M, nvn)]).astype(np.int64)
    w1 = node_table[ncand] @ f
    order1 = np.lexsort((ncand, -w1))
    expanded = np.sort(ncand[order1[:probe]])
    cand = np.concatenate([np.arange(N * M, (N + 1) * M) for N in expanded] +
                          [np.arange(nvn * M, nv)]).astype(np.int64)
    s = table_bg[cand] @ f
    corder = np.lexsort((cand, -s))
    take = min(p.topk, cand.size)
    kept = np.full(p.topk, -1, dtype=np.int64)
    kept[:take] = np.sort(cand[corder[:take]])
    tau = s[corder[p.topk - 1]] if cand.size >= p.topk else -np.inf
    f_s_norm = math.sqrt(float(f[:d] @ f[:d]))
    margin = HIER_MARGIN * math.sqrt(float(f @ f)) * t_star
    bound1 = w1[order1[probe]] + f_s_norm * r_star + margin if ncand.size > probe else -np.inf
    bound2 = w2[order2[probe]] + f_s_norm * r2_star + margin if nvs > probe else -np.inf
    certified = bool(tau > bound1 and tau > bound2) if max(bound1, bound2) > -np.inf else True
    # the gaps that float32 rounding could flip: each level's probe-th /
    # (probe+1)-th score, the kept set's k-th / (k+1)-th
    super_gap = w2[order2[probe - 1]] - w2[order2[probe]] if nvs > probe else np.inf
    node_gap = w1[order1[probe - 1]] - w1[order1[probe]] if ncand.size > probe else np.inf
    kgap = (s[corder[p.topk - 1]] - s[corder[p.topk]]) if cand.size > p.topk else np.inf
    info = {"super_expanded": sexp, "expanded": expanded, "tau": tau, "bound": max(bound1, bound2),
            "bounds": (bound1, bound2), "super_gap": super_gap, "node_gap": node_gap, "kept_gap": kgap,
            "scale": math.sqrt(float(f @ f)) * t_star}
    return kept, certified, info


def hier_route(Q: np.ndarray, stored, p: Problem, fanout: int, probe: int, escalate: bool = False,
               rows=None, levels: int = 1, list_factor=None):
    """block_idx [batch, n_q, h_kv, k], certified [batch, n_q, h_kv] (bool) and
    per-row info of the hierarchical router (bf16 problems, S = 1).

    escalate: uncertified rows take the flat top-k of all visible blocks.
    rows: optional (batch, query row) pairs; other rows stay -2 / False.
    levels: 1 (nodes over blocks) or 2 (super-nodes over the nodes as well).
    list_factor: lambda of the listed outlier blocks (one level only), or None.
    """
    if p.dtype != BF16 or p.subblocks != 1 or p.outlier:
        raise ValueError("the hierarchical router is defined on the bf16 routing table, S = 1")
    if levels not in (1, 2):
        raise ValueError("one or two tree levels")
    if list_factor is not None and (levels != 1 or not list_factor >= 1.0):
        raise ValueError("listed blocks: one tree level and a factor >= 1")
    _mu32, _sig32, table = stored
    listed = hier_listed_blocks(table, fanout, list_factor) if list_factor is not None else None
    nodes = hier_nodes(table, fanout, listed)
    supers = hier_super_nodes(nodes[0], nodes[1], nodes[3], fanout) if levels == 2 else None
    bidx = np.full((p.batch, p.n_q, p.h_kv, p.topk), -2, dtype=np.int64)
    cert = np.zeros((p.batch, p.n_q, p.h_kv), dtype=bool)
    info = {}
    if rows is None:
        rows = [(bi, i) for bi in range(p.batch) for i in range(p.n_q)]
    feats = {}
    for bi, i in rows:
        if bi not in feats:
            feats[bi] = route_features(Q[bi:bi + 1], p)[0]          # [h_kv, n_q, 2d]
        pos = p.q_offset + i
        for g in range(p.h_kv):
            f = feats[bi][g, i]
            nb_g = (nodes[0][bi, g], nodes[1][bi, g], nodes[2][bi, g], nodes[3][bi, g])
            if levels == 1:
                kept, ok, inf = hier_route_row(f, table[bi, g], nb_g, pos, p, fanout, probe,
                                               None if listed is None else listed[bi, g])
            else:
                sb_g = (supers[0][bi, g], supers[1][bi, g], supers[2][bi, g], supers[3][bi, g])
                kept, ok, inf = hier_route_row2(f, table[bi, g], nb_g, sb_g, pos, p, fanout, probe)
            if escalate and not ok:
                nv = visible_blocks(pos, p)
                kept, _gap = select_topk(table[bi, g, :nv] @ f, p.topk)
            bidx[bi, i, g] = kept
            cert[bi, i, g] = ok
            info[(bi, i, g)] = inf
    return bidx, cert, info
