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
    is part of the definition (``route_features`` / ``stored_summaries``).

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
    return mu, sig


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
    """Block scores from sub-block scores (last axis nb * S): the maximum
    over each block's S sub-blocks (identity for S = 1)."""
    S = p.subblocks
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
    nu = nv * p.subblocks                      # visible summary rows
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
