"""Plain fp64 CPU oracle of the Sol-Attn sparse attention forward.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may call it.  It shares no code with the CUDA path.

Source: "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly
Attention Sparsification" (method section: query-dependent threshold routing,
Eq. 3-5; chunk-wise streaming thresholding, Eq. 6-7; proxy-score reuse,
Eq. 8-10; batched approximation tile, Eq. 11; experiments: setup, fixed 64x64
physical blocks).  The display equations of that page did not survive text
extraction; the forms below are rebuilt from the prose around them, and each
reading is listed in the design notes:

  * pooled query / key of block j: mean of its valid tokens (Q̄_j, K̄_j);
    summed value V̂_j: sum of its valid tokens; n_j = number of valid tokens.
  * proxy logit  ŝ_ij = Q̄_i · K̄_j / sqrt(d).
  * row mean / variance from the pooled-key moments:
        m = (1/N) Σ_j K̄_j,   Σ_K = (1/N) Σ_j (K̄_j - m)(K̄_j - m)^T,
        μ_i = Q̄_i · m / sqrt(d),   σ_i^2 = Q̄_i^T Σ_K Q̄_i / d   (population).
  * τ_i = μ_i + β σ_i;  S_i = {j : ŝ_ij >= τ_i};  U_i = the rest.
    β = -inf selects every block, β = +inf selects none.
  * for a query token r of block i (logits scaled by 1/sqrt(d)):
        D_r = Σ_{j∈S_i} Σ_{k∈j} exp(q_r·k_k) + Σ_{j∈U_i} n_j exp(q_r·K̄_j)
        N_r = Σ_{j∈S_i} Σ_{k∈j} exp(q_r·k_k) v_k + Σ_{j∈U_i} exp(q_r·K̄_j) V̂_j
        O_r = N_r / D_r        (0 when D_r = 0, which only exact-only can reach).
    The approximation uses the per-token logit q_r·K̄_j (the B x 1 centre of the
    zeroth-order Taylor term), not the block-level ŝ_ij.
  * optional first-order term (taylor_order=1): the expansion of a skipped
    block's exponential scores around that same centre c_r = q_r·K̄_j/sqrt(d),
        exp(s_rk) ≈ exp(c_r) (1 + (s_rk - c_r)),
    whose added term exp(c_r)(s_rk - c_r) enters D and N like an exact score
    (its row sum over the block is zero, so only N changes).  The pages keep
    the zeroth order only; the first order is this build's extension.

Every array is float64.  Matmuls and reductions are library primitives; there
is no blocking, fusion or reordering beyond the definitions above.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np

__all__ = [
    "pool_blocks", "proxy_row", "proxy_logits", "key_moments", "row_stats_from_moments",
    "row_stats_bruteforce", "thresholds", "select_global", "select_streaming",
    "approx_logits", "sol_attn_head",
]


def _nblocks(L: int, block: int) -> int:
    return -(-L // block)


def pool_blocks(x: np.ndarray, block: int = 64):
    """Block pooling of one (batch, head) slice x [L, d].

    Returns (means [N, d], sums [N, d], counts n [N]).  Block j covers tokens
    [j*block, min((j+1)*block, L)); a ragged last block is pooled over its valid
    tokens only.  Means give Q̄ / K̄ (method: threshold routing, block-proxy
    logits of Eq. 3); sums give the summed value V̂_j (method: proxy-score reuse,
    definition before Eq. 9).
    """
    L, d = x.shape
    N = _nblocks(L, block)
    n = np.array([min(block, L - j * block) for j in range(N)], dtype=np.int64)
    sums = np.stack([x[j * block: j * block + n[j]].sum(axis=0) for j in range(N)])
    means = sums / n[:, None]
    return means, sums, n


def proxy_row(qbar_i: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """ŝ_ij = Q̄_i · K̄_j / sqrt(d) for one query block against a set of pooled keys
    (method: threshold routing, Eq. 3).  Each dot product is an elementwise
    product summed over d, so a given (i, j) pair rounds the same way whichever
    subset of keys it is evaluated with."""
    d = qbar_i.shape[-1]
    return (kbar * qbar_i[None, :]).sum(axis=-1) / math.sqrt(d)


def proxy_logits(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """Full N x N proxy map (the oracle may materialise it; the method does not)."""
    return np.stack([proxy_row(qbar[i], kbar) for i in range(qbar.shape[0])])


def key_moments(kbar: np.ndarray):
    """First and second (central) moments of the pooled keys (method: threshold
    routing, Eq. 5): m = mean_j K̄_j and Σ_K = mean_j (K̄_j - m)(K̄_j - m)^T."""
    N = kbar.shape[0]
    m = kbar.mean(axis=0)
    kc = kbar - m[None, :]
    sigma_k = kc.T @ kc / N
    return m, sigma_k


def row_stats_from_moments(qbar: np.ndarray, m: np.ndarray, sigma_k: np.ndarray):
    """μ_i = Q̄_i·m/sqrt(d), σ_i = sqrt(Q̄_i^T Σ_K Q̄_i / d) without forming the proxy
    map (method: threshold routing, Eq. 5; O(Ld + Nd^2) time, O(d^2) memory)."""
    d = qbar.shape[1]
    mu = qbar @ m / math.sqrt(d)
    var = np.einsum("id,de,ie->i", qbar, sigma_k, qbar) / d
    sigma = np.sqrt(np.maximum(var, 0.0))
    return mu, sigma


def row_stats_bruteforce(s_hat: np.ndarray):
    """Row mean and population standard deviation of a materialised proxy map."""
    return s_hat.mean(axis=1), s_hat.std(axis=1)


def thresholds(mu: np.ndarray, sigma: np.ndarray, beta: float) -> np.ndarray:
    """τ_i = μ_i + β σ_i (method: threshold routing, Eq. 4).  β = -inf gives
    τ = -inf (every block selected), β = +inf gives τ = +inf (none)."""
    if math.isinf(beta):
        return np.full_like(mu, beta)
    return mu + beta * sigma


def select_global(s_hat_row: np.ndarray, tau_i: float) -> np.ndarray:
    """S_i as a boolean row: ŝ_ij >= τ_i (method: threshold routing, Eq. 4)."""
    return s_hat_row >= tau_i


def select_streaming(qbar_i: np.ndarray, kbar: np.ndarray, tau_i: float, chunk: int):
    """Chunk-wise streaming thresholding (method: Eq. 6-7).

    The pooled keys are cut into T = ceil(N/C) chunks; each chunk's proxy scores
    are compared with τ_i as soon as they are produced.  Returns the per-chunk
    selected index lists S_i^(t); their union is S_i."""
    N = kbar.shape[0]
    T = -(-N // chunk)
    per_chunk = []
    for t in range(T):
        lo, hi = t * chunk, min((t + 1) * chunk, N)
        s_t = proxy_row(qbar_i, kbar[lo:hi])
        per_chunk.append([lo + c for c in range(hi - lo) if s_t[c] >= tau_i])
    return per_chunk


def approx_logits(q_rows: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """Token-to-block score tile q_r · K̄_j / sqrt(d) (method: proxy-score reuse,
    Eq. 8 zeroth-order centre; Eq. 11 batched tile)."""
    d = q_rows.shape[1]
    return q_rows @ kbar.T / math.sqrt(d)


def sol_attn_head(q, k, v, beta: float, block: int = 64, *, exact_only: bool = False,
                  rows: Optional[list] = None, sel_override: Optional[np.ndarray] = None,
                  taylor_order: int = 0):
    """Sol-Attn forward for one (batch, head) slice, non-streaming, in fp64.

    q, k, v: [L, d] float64 (callers widen the bf16 inputs exactly).
    rows: query-block indices to evaluate (default: all).  Output rows of other
    blocks are left as NaN.
    sel_override: optional [N, N] boolean selection used instead of the
    threshold test (to evaluate a different but equally valid selection).
    exact_only: keep-or-drop sparse attention on the same selection
    (ablation: exact-only vs exact-or-approx, Fig. 7).
    taylor_order: 0 (the method: zeroth-order term of Eq. 8) or 1 (adds the
    first-order term of the same expansion for every unselected block).

    Returns dict with O [L, d], counts [N], sel [N, N] (rows evaluated),
    qbar, kbar, vhat, n, mu, sigma, tau.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    L, d = q.shape
    N = _nblocks(L, block)
    qbar, _, nq = pool_blocks(q, block)
    kbar, _, n = pool_blocks(k, block)
    _, vhat, _ = pool_blocks(v, block)
    m, sigma_k = key_moments(kbar)
    mu, sigma = row_stats_from_moments(qbar, m, sigma_k)
    tau = thresholds(mu, sigma, beta)
    if rows is None:
        rows = list(range(N))
    O = np.full((L, d), np.nan)
    sel = np.zeros((N, N), dtype=bool)
    counts = np.zeros(N, dtype=np.int64)
    scale = 1.0 / math.sqrt(d)
    for i in rows:
        if sel_override is not None:
            s_i = np.asarray(sel_override[i], dtype=bool)
        else:
            s_i = select_global(proxy_row(qbar[i], kbar), tau[i])
        sel[i] = s_i
        counts[i] = int(s_i.sum())
        lo, hi = i * block, min((i + 1) * block, L)
        qi = q[lo:hi]
        S = np.nonzero(s_i)[0]
        U = np.nonzero(~s_i)[0]
        key_idx = np.concatenate([np.arange(j * block, min((j + 1) * block, L)) for j in S]) \
            if len(S) else np.zeros(0, dtype=np.int64)
        e = qi @ k[key_idx].T * scale                         # exact logits  [n_i, keys]
        if exact_only or len(U) == 0:
            a = np.zeros((qi.shape[0], 0))
            U = U[:0]
        else:
            a = approx_logits(qi, kbar[U])                     # approx logits [n_i, |U|]
        both = np.concatenate([e, a], axis=1)
        if both.shape[1] == 0:
            O[lo:hi] = 0.0
            continue
        M = both.max(axis=1, keepdims=True)
        pe = np.exp(e - M)
        pa = np.exp(a - M)
        D = pe.sum(axis=1) + (pa * n[U][None, :]).sum(axis=1)
        Nn = pe @ v[key_idx] + pa @ vhat[U]
        if taylor_order >= 1:
            # first-order term exp(c)(S_j - c) of each skipped block j, with the
            # block's exact scores S_j and the centre c = a[:, u] broadcast over keys
            for u, j in enumerate(U):
                kj = np.arange(j * block, min((j + 1) * block, L))
                resid = qi @ k[kj].T * scale - a[:, u:u + 1]
                term = pa[:, u:u + 1] * resid
                D = D + term.sum(axis=1)
                Nn = Nn + term @ v[kj]
        O[lo:hi] = Nn / D[:, None]
    return dict(O=O, counts=counts, sel=sel, qbar=qbar, kbar=kbar, vhat=vhat, n=n,
                mu=mu, sigma=sigma, tau=tau, m=m, sigma_k=sigma_k)
