"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test names the passage of "Sol-Attn: Accelerating Video Generation
Inference via On-the-Fly Attention Sparsification" it follows.  Together they
are chosen so that a plausible slip in the oracle (wrong scale, a dropped
multiplicity n_j, mean instead of sum for V̂, a reversed threshold test,
variance instead of standard deviation, a chunk-boundary off-by-one, a
mis-pooled ragged tail) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import (approx_logits, key_moments, pool_blocks, proxy_logits, proxy_row,
                    row_stats_bruteforce, row_stats_from_moments, select_global,
                    select_streaming, sol_attn_head, thresholds)
from synth import WORKLOADS, bf16_bits_to_f64, custom_fourier, fourier_inputs, gauss_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _fourier_head(grid, d, amp=2.0, seed=7):
    q, k, v = custom_fourier(1, 1, grid, d, amp, seed)
    return bf16_bits_to_f64(q[0, 0]), bf16_bits_to_f64(k[0, 0]), bf16_bits_to_f64(v[0, 0])


def _sdpa(q, k, v):
    """Library softmax attention in fp64 (torch CPU)."""
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v))[0, 0].numpy()


def _rel_l2(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


# --- block pooling (method: threshold routing, Eq. 3; proxy-score reuse, V̂) ------------

def test_pool_constant_blocks_and_ragged_tail():
    L, d, blk = 130, 5, 64                      # blocks of 64, 64 and a 2-token tail
    x = np.zeros((L, d))
    consts = np.array([[1.5, -2.0, 0.25, 3.0, 7.0], [0.5, 1.0, -4.0, 2.0, 0.0], [9.0, -1.0, 1.0, 1.0, 2.5]])
    for j in range(3):
        x[j * blk: min((j + 1) * blk, L)] = consts[j]
    means, sums, n = pool_blocks(x, blk)
    assert list(n) == [64, 64, 2]
    np.testing.assert_array_equal(means, consts)
    np.testing.assert_array_equal(sums, consts * np.array([64, 64, 2])[:, None])


# --- moments (method: threshold routing, Eq. 5 and the O(Ld + Nd^2) remark) --------------

@pytest.mark.parametrize("kind", ["fourier", "gauss", "offset"])
def test_moment_stats_equal_bruteforce(kind):
    if kind == "gauss":
        q, k, _ = gauss_inputs(1, 1, 64 * 40 + 17, 64, seed=3)
        q, k = bf16_bits_to_f64(q[0, 0]), bf16_bits_to_f64(k[0, 0])
    else:
        q, k, _ = _fourier_head((3, 20, 31), 128, amp=3.0)
        if kind == "offset":            # large common offset: cancellation-prone
            k = k + 40.0
    qbar, _, _ = pool_blocks(q)
    kbar, _, _ = pool_blocks(k)
    s = proxy_logits(qbar, kbar)
    mu_b, sd_b = row_stats_bruteforce(s)            # numpy mean / population std
    m, sig = key_moments(kbar)
    mu_m, sd_m = row_stats_from_moments(qbar, m, sig)
    scale = np.abs(s).max()
    np.testing.assert_allclose(mu_m, mu_b, rtol=0, atol=1e-10 * scale)
    np.testing.assert_allclose(sd_m, sd_b, rtol=1e-9, atol=1e-10 * scale)


# --- threshold + Gaussian calibration (method: Eq. 4, Fig. 3) ------------------------------

def _golden_density():
    rows = []
    with open(os.path.join(GOLDEN, "gaussian_density.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                b, r = line.split()
                rows.append((float(b), float(r)))
    return rows


def test_golden_density_table_is_the_gaussian_tail():
    for beta, rho in _golden_density():
        assert abs(0.5 * math.erfc(beta / math.sqrt(2.0)) - rho) < 6e-5


def test_density_matches_gaussian_reference():
    # iid Gaussian Q, K: given Q̄_i the proxy row is Gaussian over j, so the mean
    # selected density is 1 - Phi(beta) up to O(1/sqrt(N)) per row.
    L, d = 64 * 512, 64
    q, k, _ = gauss_inputs(1, 1, L, d, seed=11)
    q, k = bf16_bits_to_f64(q[0, 0]), bf16_bits_to_f64(k[0, 0])
    qbar, _, _ = pool_blocks(q)
    kbar, _, _ = pool_blocks(k)
    m, sig = key_moments(kbar)
    mu, sd = row_stats_from_moments(qbar, m, sig)
    s = proxy_logits(qbar, kbar)
    for beta, rho in _golden_density():
        tau = thresholds(mu, sd, beta)
        dens = np.mean([select_global(s[i], tau[i]).mean() for i in range(len(tau))])
        assert abs(dens - rho) < 0.01, (beta, dens, rho)


def test_infinite_beta_selects_all_or_none():
    q, k, _ = _fourier_head((2, 8, 40), 64)
    qbar, _, _ = pool_blocks(q)
    kbar, _, _ = pool_blocks(k)
    mu, sd = row_stats_from_moments(qbar, *key_moments(kbar))
    s = proxy_logits(qbar, kbar)
    assert all(select_global(s[i], t).all() for i, t in enumerate(thresholds(mu, sd, -math.inf)))
    assert not any(select_global(s[i], t).any() for i, t in enumerate(thresholds(mu, sd, math.inf)))


# --- streaming thresholding (method: Eq. 6-7, "recovers the same block set") ---------------

def test_streaming_selection_equals_global():
    q, k, _ = _fourier_head((2, 16, 45), 64)          # L = 1440, N = 23 (ragged)
    qbar, _, _ = pool_blocks(q)
    kbar, _, _ = pool_blocks(k)
    N = kbar.shape[0]
    mu, sd = row_stats_from_moments(qbar, *key_moments(kbar))
    for beta in (0.0, 0.75, 1.0, 1.5):
        tau = thresholds(mu, sd, beta)
        for C in (1, 3, 4, 7, 16, N, N + 5):
            for i in range(N):
                chunks = select_streaming(qbar[i], kbar, tau[i], C)
                assert len(chunks) == -(-N // C)
                for t, lst in enumerate(chunks):
                    assert all(t * C <= j < min((t + 1) * C, N) for j in lst)
                union = sorted(j for lst in chunks for j in lst)
                glob = list(np.nonzero(select_global(proxy_row(qbar[i], kbar), tau[i]))[0])
                assert union == glob


# --- approximation tile (method: Eq. 11, column means recover the routing scores) --------

def test_tile_column_means_equal_proxy_scores():
    q, k, _ = _fourier_head((2, 10, 33), 128)
    qbar, _, _ = pool_blocks(q)
    kbar, _, _ = pool_blocks(k)
    for i in range(qbar.shape[0]):
        rows = q[i * 64: min((i + 1) * 64, q.shape[0])]
        tile = approx_logits(rows, kbar)
        np.testing.assert_allclose(tile.mean(axis=0), proxy_row(qbar[i], kbar), rtol=0, atol=1e-12)


# --- combined numerator / denominator (method: Eq. 8-10) -------------------------------

@pytest.mark.parametrize("L", [1024, 1000, 65])
def test_select_all_is_softmax_attention(L):
    q, k, v = _fourier_head((1, 1, L), 64)
    r = sol_attn_head(q, k, v, -math.inf)
    assert (r["counts"] == r["n"].shape[0]).all()
    np.testing.assert_allclose(r["O"], _sdpa(q, k, v), rtol=0, atol=1e-12)
    r2 = sol_attn_head(q, k, v, -math.inf, exact_only=True)
    np.testing.assert_allclose(r2["O"], _sdpa(q, k, v), rtol=0, atol=1e-12)


@pytest.mark.parametrize("L", [1024, 1000])
def test_block_constant_keys_reduce_to_dense(L):
    # With every key equal to its block's mean, the zeroth-order term is exact:
    # the output equals dense attention for any beta (Eq. 8 with a zero residual).
    q, k, v = _fourier_head((1, 1, L), 64, amp=2.5, seed=19)
    kbar, _, n = pool_blocks(k)
    kc = np.repeat(kbar, n, axis=0)
    dense = _sdpa(q, kc, v)
    seen_mixed = False
    for beta in (-math.inf, 0.0, 0.5, 1.0, 2.0, math.inf):
        r = sol_attn_head(q, kc, v, beta)
        np.testing.assert_allclose(r["O"], dense, rtol=0, atol=1e-12)
        seen_mixed |= bool(((r["counts"] > 0) & (r["counts"] < len(n))).any())
    assert seen_mixed


def test_select_none_is_pooled_softmax_with_multiplicity():
    # beta = +inf: every block approximated, i.e. softmax over the N pooled keys
    # with log-multiplicity log n_j applied to the mean values V̄_j.
    L, d = 1000, 64
    q, k, v = _fourier_head((1, 1, L), d, seed=23)
    N = -(-L // 64)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    pad = N * 64 - L
    kp = torch.cat([tk, torch.zeros(pad, d, dtype=torch.float64)])
    vp = torch.cat([tv, torch.zeros(pad, d, dtype=torch.float64)])
    n = torch.tensor([64] * (N - 1) + [64 - pad], dtype=torch.float64)
    kbar = kp.view(N, 64, d).sum(1) / n[:, None]
    vbar = vp.view(N, 64, d).sum(1) / n[:, None]
    logits = tq @ kbar.T / math.sqrt(d) + torch.log(n)[None, :]
    expect = torch.softmax(logits, dim=1) @ vbar
    r = sol_attn_head(q, k, v, math.inf)
    assert (r["counts"] == 0).all()
    np.testing.assert_allclose(r["O"], expect.numpy(), rtol=0, atol=1e-12)


def test_exact_only_with_nothing_selected_outputs_zero():
    q, k, v = _fourier_head((1, 1, 300), 64)
    r = sol_attn_head(q, k, v, math.inf, exact_only=True)
    assert (r["O"] == 0).all()


def test_key_shift_invariance():
    # K -> K + c shifts every logit of a row by the same q·c: selection and
    # output are unchanged (mu_i moves with the scores, sigma_i does not).
    q, k, v = _fourier_head((2, 8, 50), 64, seed=29)
    c = np.random.default_rng(0).normal(0, 2.0, size=(1, 64))
    for beta in (0.5, 1.0):
        a = sol_attn_head(q, k, v, beta)
        b = sol_attn_head(q, k + c, v, beta)
        np.testing.assert_array_equal(a["sel"], b["sel"])
        np.testing.assert_allclose(a["O"], b["O"], rtol=0, atol=1e-10)


def test_key_block_permutation_invariance():
    L = 64 * 12                                   # no ragged tail: blocks are interchangeable
    q, k, v = _fourier_head((1, 1, L), 64, seed=31)
    perm = np.random.default_rng(1).permutation(12)
    idx = np.concatenate([np.arange(p * 64, (p + 1) * 64) for p in perm])
    for beta in (0.25, 1.0):
        a = sol_attn_head(q, k, v, beta)
        b = sol_attn_head(q, k[idx], v[idx], beta)
        np.testing.assert_array_equal(a["sel"][:, perm], b["sel"])
        np.testing.assert_allclose(a["O"], b["O"], rtol=0, atol=1e-12)


def test_approximation_reduces_error_vs_exact_only():
    # Ablation (Fig. 7): under identical indices, exact-or-approx has a lower
    # relative l2 error against dense attention than keep-or-drop.
    wl = WORKLOADS["small"]
    q, k, v = fourier_inputs(wl, heads=[0])
    q, k, v = (bf16_bits_to_f64(x[0, 0]) for x in (q, k, v))
    dense = _sdpa(q, k, v)
    for beta in (0.5, 1.0, 1.5):
        approx = sol_attn_head(q, k, v, beta)["O"]
        exact = sol_attn_head(q, k, v, beta, exact_only=True)["O"]
        assert _rel_l2(approx, dense) < _rel_l2(exact, dense)


def test_sel_override_reproduces_threshold_selection():
    q, k, v = _fourier_head((2, 8, 40), 64)
    a = sol_attn_head(q, k, v, 1.0)
    b = sol_attn_head(q, k, v, 1.0, sel_override=a["sel"])
    np.testing.assert_array_equal(a["O"], b["O"])


# --- output structure (method: Eq. 9-10, the normalised sum over exact and approximated keys) ---

@pytest.mark.parametrize("beta", [0.5, 1.0, math.inf])
def test_constant_values_give_that_constant(beta):
    # With V = c everywhere, V̂_j = n_j c, so every output row is
    # (Σ e^s c + Σ_j n_j e^a c) / (Σ e^s + Σ_j n_j e^a) = c exactly: the weights
    # are normalised, and n_j appears on both sides (a ragged 37-token tail
    # included).  Dropping n_j from either side, or pooling V̂ as a mean, breaks it.
    q, k, _ = _fourier_head((1, 1, 64 * 9 + 37), 64, seed=41)
    c = np.array([0.75, -2.5] * 32)
    v = np.tile(c, (q.shape[0], 1))
    out = sol_attn_head(q, k, v, beta)["O"]
    np.testing.assert_allclose(out, np.tile(c, (q.shape[0], 1)), rtol=0, atol=1e-12)


def test_output_is_linear_in_values():
    # The selection and every weight depend on Q and K only, so the output is
    # linear in V (V̂ is a linear pooling of V).
    q, k, v1 = _fourier_head((1, 2, 300), 64, seed=43)
    v2 = np.random.default_rng(2).normal(size=v1.shape)
    for beta in (0.5, 1.0):
        o1 = sol_attn_head(q, k, v1, beta)["O"]
        o2 = sol_attn_head(q, k, v2, beta)["O"]
        o12 = sol_attn_head(q, k, 2.0 * v1 - 0.5 * v2, beta)["O"]
        np.testing.assert_allclose(o12, 2.0 * o1 - 0.5 * o2, rtol=0, atol=1e-10)


def test_query_key_rescaling_invariance():
    # (Q, K) -> (c Q, K / c) leaves every exact, proxy and approximation logit
    # unchanged, and with them μ_i, σ_i, τ_i: same selection, same output.
    q, k, v = _fourier_head((2, 8, 50), 64, seed=47)
    for beta in (0.5, 1.0):
        a = sol_attn_head(q, k, v, beta)
        b = sol_attn_head(4.0 * q, k / 4.0, v, beta)
        np.testing.assert_array_equal(a["sel"], b["sel"])
        np.testing.assert_allclose(a["O"], b["O"], rtol=0, atol=1e-10)


# --- first-order term of the expansion (method: proxy-score reuse, Eq. 8; the pages keep
# --- only the zeroth order, the first order is this build's extension) -----------------

def _blocky_keys(L, d, seed, eps):
    """Keys equal to their block's mean plus eps times a fixed zero-mean-per-block residual."""
    q, k, v = _fourier_head((1, 1, L), d, amp=2.5, seed=seed)
    kbar, _, n = pool_blocks(k)
    noise = np.random.default_rng(seed + 1).standard_normal(k.shape)
    for j in range(len(n)):
        sl = slice(64 * j, 64 * j + n[j])
        noise[sl] -= noise[sl].mean(axis=0)
    return q, np.repeat(kbar, n, axis=0), noise, v


@pytest.mark.parametrize("beta", [0.5, 1.0, 1.5])
def test_first_order_error_falls_with_the_square_of_the_key_spread(beta):
    # With keys K̄_j + eps R (R zero-mean within each block) the skipped blocks'
    # scores deviate from the centre by O(eps).  Dropping everything after the
    # zeroth order leaves an O(eps) error in the numerator; keeping the first
    # order leaves O(eps^2).  Halving eps must halve the first error and quarter
    # the second (a missing, mis-signed or mis-centred first-order term fails).
    q, base, noise, v = _blocky_keys(64 * 12 + 37, 64, 19, 0.0)
    errs = {}
    for eps in (0.1, 0.05):
        kk = base + eps * noise
        dense = _sdpa(q, kk, v)
        for order in (0, 1):
            errs[order, eps] = _rel_l2(sol_attn_head(q, kk, v, beta, taylor_order=order)["O"], dense)
    r0 = errs[0, 0.1] / errs[0, 0.05]
    r1 = errs[1, 0.1] / errs[1, 0.05]
    assert 1.8 < r0 < 2.25, r0
    assert 3.6 < r1 < 4.4, r1
    assert errs[1, 0.05] < errs[0, 0.05] / 4


@pytest.mark.parametrize("L", [1024, 1000])
def test_first_order_term_vanishes_on_block_constant_keys(L):
    # Keys equal to their block mean: every score of a skipped block equals its
    # centre, the first-order term is zero and the output is dense attention.
    q, k, v = _fourier_head((1, 1, L), 64, amp=2.5, seed=19)
    kbar, _, n = pool_blocks(k)
    kc = np.repeat(kbar, n, axis=0)
    dense = _sdpa(q, kc, v)
    for beta in (0.0, 1.0, math.inf):
        r = sol_attn_head(q, kc, v, beta, taylor_order=1)
        np.testing.assert_allclose(r["O"], dense, rtol=0, atol=1e-12)


def test_first_order_with_every_block_selected_is_softmax_attention():
    q, k, v = _fourier_head((1, 1, 1000), 64)
    r = sol_attn_head(q, k, v, -math.inf, taylor_order=1)
    np.testing.assert_allclose(r["O"], _sdpa(q, k, v), rtol=0, atol=1e-12)
