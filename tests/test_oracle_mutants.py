"""Planted mistakes in the oracle must fail its pins.

Each mutant below is a plausible slip in the fp64 oracle (written on the CPU,
into a temporary copy of the repository).  The pins in test_oracle_pins.py are
run against every mutant; each must make at least one pin fail.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "sol_attn_oracle.py")

MUTANTS = {
    "summed_value_is_mean": ("_, vhat, _ = pool_blocks(v, block)", "vhat, _, _ = pool_blocks(v, block)"),
    "multiplicity_dropped": ("(pa * n[U][None, :]).sum(axis=1)", "pa.sum(axis=1)"),
    "variance_for_std": ("sigma = np.sqrt(np.maximum(var, 0.0))", "sigma = np.maximum(var, 0.0)"),
    "threshold_reversed": ("return s_hat_row >= tau_i", "return s_hat_row <= tau_i"),
    "proxy_scale_1_over_d": ("return (kbar * qbar_i[None, :]).sum(axis=-1) / math.sqrt(d)",
                             "return (kbar * qbar_i[None, :]).sum(axis=-1) / d"),
    "approx_scale_1_over_d": ("return q_rows @ kbar.T / math.sqrt(d)", "return q_rows @ kbar.T / d"),
    "sample_covariance": ("sigma_k = kc.T @ kc / N", "sigma_k = kc.T @ kc / (N - 1)"),
    "ragged_tail_full_count": ("n = np.array([min(block, L - j * block) for j in range(N)], dtype=np.int64)",
                               "n = np.array([block for j in range(N)], dtype=np.int64)"),
    "chunk_bound_off_by_one": ("lo, hi = t * chunk, min((t + 1) * chunk, N)",
                               "lo, hi = t * chunk, min((t + 1) * chunk, N - 1)"),
    "mean_sign": ("mu = qbar @ m / math.sqrt(d)", "mu = -qbar @ m / math.sqrt(d)"),
    "threshold_minus_beta": ("return mu + beta * sigma", "return mu - beta * sigma"),
    "approx_block_level_logit": ("a = approx_logits(qi, kbar[U])",
                                 "a = np.repeat(approx_logits(qbar[i:i+1], kbar[U]), qi.shape[0], axis=0)"),
    "first_order_sign": ("term = pa[:, u:u + 1] * resid", "term = -pa[:, u:u + 1] * resid"),
    "first_order_block_level_centre": ("resid = qi @ k[kj].T * scale - a[:, u:u + 1]",
                                       "resid = qi @ k[kj].T * scale - proxy_row(qbar[i], kbar[j:j + 1])[None, :]"),
    "first_order_dropped_from_numerator": ("Nn = Nn + term @ v[kj]", "Nn = Nn"),
}


@pytest.fixture(scope="module")
def scratch(tmp_path_factory):
    d = tmp_path_factory.mktemp("mutant_repo")
    for sub in ("oracle", "synth", "tests"):
        shutil.copytree(os.path.join(ROOT, sub), os.path.join(d, sub),
                        ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutants.py", "test_*gpu*"))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), d)
    return str(d)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(scratch, name):
    good, bad = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(good) == 1, name
    with open(os.path.join(scratch, "oracle", "sol_attn_oracle.py"), "w") as f:
        f.write(src.replace(good, bad))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_oracle_pins.py"], cwd=scratch, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode != 0, f"mutant {name} survived:\n{r.stdout[-2000:]}"
