"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
identical seeded bf16 inputs, for the five workload shapes and the edge cases.

"Sol-Attn: Accelerating Video Generation Inference via On-the-Fly Attention
Sparsification": masks follow Eq. 4 / Eq. 6-7, outputs Eq. 9-10."""
import math

import numpy as np
import pytest

import block_sparse_attention_moments_b200 as sa
from parity_util import (MAX_ABS, MAX_ABS_FIRST_ORDER, Report, check_counts, check_full_masks, compare_head,
                         debug_numpy, run_gpu)
from synth import (WORKLOADS, custom_fourier, fourier_inputs, gauss_inputs, near_block_constant_keys,
                   offset_inputs, ramp_inputs)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    sa.lib()


def _full_check(qb, kb, vb, beta, chunk, flags=0, heads=None, rows=None, mask_heads=(), count_heads=()):
    """Outputs of `heads` (all by default) on `rows` (all by default) against
    the oracle, per head; every row's mask of `mask_heads`; the counts of
    `count_heads` against the oracle's thresholds."""
    out, dbg, counts = run_gpu(qb, kb, vb, beta, chunk, flags=flags)
    sel = dbg.selection().cpu().numpy()
    dn = debug_numpy(dbg)
    rep = Report(MAX_ABS_FIRST_ORDER if flags & sa.FLAG_FIRST_ORDER else MAX_ABS)
    B, H = qb.shape[:2]
    for bh in (range(B * H) if heads is None else heads):
        b, h = divmod(bh, H)
        compare_head(rep, qb, kb, vb, b, h, beta, out, sel, counts, rows=rows,
                     exact_only=bool(flags & sa.FLAG_EXACT_ONLY), dbg=dn,
                     taylor_order=1 if flags & sa.FLAG_FIRST_ORDER else 0)
    if not math.isinf(beta):
        for bh in mask_heads:
            check_full_masks(rep, qb, kb, *divmod(bh, H), beta, sel, counts)
        for bh in count_heads:
            check_counts(qb, kb, *divmod(bh, H), beta, counts)
    print(rep)
    rep.publish()
    rep.check()
    return out, sel, rep


@pytest.mark.parametrize("beta", [1.0, 0.5, 1.5, -math.inf, math.inf])
def test_tiny_shape(beta):
    wl = WORKLOADS["tiny"]
    qb, kb, vb = fourier_inputs(wl)
    _full_check(qb, kb, vb, beta, wl.chunk)


@pytest.mark.parametrize("beta", [0.5, 1.0, 1.5, -math.inf, 0.0, -0.5])
def test_small_shape(beta):
    wl = WORKLOADS["small"]
    qb, kb, vb = fourier_inputs(wl)
    _full_check(qb, kb, vb, beta, wl.chunk)


@pytest.mark.parametrize("beta", [-math.inf, 0.5, 1.0])
def test_running_maximum_rises_along_the_walk(beta):
    # Key norms grow along the sequence, so most rows meet their largest logits
    # late in their walk: the running maximum rises by tens of doublings, and
    # the rare path (raise m, rescale O, recompute P from S) runs on most rows.
    # The softmax rows are nearly one-hot here, so O is about one row of V; V is
    # scaled by 1/4 to keep |O| in the range of the other workloads (with unit V,
    # |O| reaches 4.9, where one bf16 rounding of the output alone is 0.016).
    qb, kb, vb = ramp_inputs(1, 2, 4096, 128, 2.0, 0.25, 4.0, seed=91, v_amp=0.25)
    _full_check(qb, kb, vb, beta, 16)


@pytest.mark.parametrize("sign", [-1.0, 1.0])
@pytest.mark.parametrize("beta", [-math.inf, 1.0])
def test_logits_far_from_zero(sign, beta):
    # Every logit near -141 (or +141) nats, about -204 (+204) doublings: against
    # the provisional reference 0 of a row's first tile every 2^y underflows to
    # 0 (or overflows to inf), so the row's first m must come from its exact
    # maximum; softmax is shift-invariant, so the result is ordinary attention.
    qb, kb, vb = offset_inputs(1, 2, 2048, 128, 40.0, sign, 0.1, seed=93)
    _full_check(qb, kb, vb, beta, 8)


def test_chunk_size_does_not_change_the_result():
    # experiments: setup — C affects efficiency, not the output
    wl = WORKLOADS["small"]
    qb, kb, vb = fourier_inputs(wl)
    ref_out, ref_sel, _ = _full_check(qb, kb, vb, 1.0, wl.chunk)
    for C in (1, 3, 7, 32, 64, 100, 500):
        out, sel, _ = _full_check(qb, kb, vb, 1.0, C)
        assert (sel == ref_sel).all()
        assert np.abs(out - ref_out).max() <= 2e-2


@pytest.mark.parametrize("chunk", [1100, 4096])
def test_window_wider_than_one_listing_pass(chunk):
    # The tile walk lists a window's union blocks 1024 at a time; a window of
    # C > 1024 pooled keys (N = 2304 here, so C = 4096 puts every block in one
    # window) needs several passes and a block carried between them.
    qb, kb, vb = custom_fourier(1, 2, (9, 64, 256), 128, 3.0, seed=91)
    N = qb.shape[2] // 64
    rows = [0, 1, 700, 1151, 1152, N - 2, N - 1]
    ref_out, ref_sel, _ = _full_check(qb, kb, vb, 1.0, 64, rows=rows)
    out, sel, _ = _full_check(qb, kb, vb, 1.0, chunk, rows=rows, mask_heads=[1])
    assert (sel == ref_sel).all()
    assert np.abs(out - ref_out).max() <= 2e-2


def test_select_all_flag_equals_dense_beta():
    wl = WORKLOADS["small"]
    qb, kb, vb = fourier_inputs(wl)
    a, _, _ = run_gpu(qb, kb, vb, 1.0, wl.chunk, flags=sa.FLAG_SELECT_ALL, debug=False)
    b, _, _ = run_gpu(qb, kb, vb, -math.inf, wl.chunk, debug=False)
    assert np.array_equal(a, b)
    _full_check(qb, kb, vb, -math.inf, wl.chunk, flags=sa.FLAG_SELECT_ALL)


@pytest.mark.parametrize("beta", [0.5, 1.0, math.inf])
def test_exact_only_flag(beta):
    wl = WORKLOADS["small"]
    qb, kb, vb = fourier_inputs(wl)
    _full_check(qb, kb, vb, beta, wl.chunk, flags=sa.FLAG_EXACT_ONLY)


def test_image_shape():
    wl = WORKLOADS["image"]
    qb, kb, vb = fourier_inputs(wl)
    B, H = wl.B, wl.H
    # three heads in full, and sampled query blocks of every other head
    full = [0, H + 7, B * H - 1]
    _full_check(qb, kb, vb, 1.0, wl.chunk, heads=full)
    rng = np.random.default_rng(5)
    rows = sorted(set(rng.integers(0, wl.N, size=6).tolist()) | {0, wl.N - 1})
    others = [bh for bh in range(B * H) if bh not in full]
    # every other head: sampled outputs of every fifth, every row's mask of
    # every fifth, the counts of all
    _full_check(qb, kb, vb, 1.0, wl.chunk, heads=others[::5], rows=rows, mask_heads=others[2::5],
                count_heads=range(B * H))


_VIDEO = {}


def _video_inputs(name):
    if name not in _VIDEO:
        _VIDEO.clear()
        _VIDEO[name] = fourier_inputs(WORKLOADS[name])
    return _VIDEO[name]


@pytest.mark.parametrize("name,beta", [("wan", 1.0), ("wan", 0.75), ("wan", 1.5), ("hunyuan", 1.0),
                                       ("hunyuan", 0.75), ("hunyuan", 1.5), ("hunyuan", -math.inf)])
def test_video_shapes_sampled(name, beta):
    # full-size launch (the bench's configuration); oracle outputs on sampled
    # query blocks of sampled heads, always including the ragged last block;
    # every row's mask of those heads; at beta = 1 the counts of every head
    wl = WORKLOADS[name]
    qb, kb, vb = _video_inputs(name)
    rng = np.random.default_rng(11)
    heads = sorted(set(rng.integers(0, wl.B * wl.H, size=3).tolist()) | {wl.B * wl.H - 1})
    rows = sorted(set(rng.integers(0, wl.N, size=4).tolist()) | {0, wl.N - 2, wl.N - 1})
    _full_check(qb, kb, vb, beta, wl.chunk, heads=heads, rows=rows, mask_heads=heads,
                count_heads=range(wl.B * wl.H) if beta == 1.0 else ())


@pytest.mark.parametrize("shape", ["tiny", "small"])
@pytest.mark.parametrize("beta", [0.75, 1.0, 1.5])
def test_mixed_selection_with_heavy_approximation(shape, beta):
    # Keys nearly constant within each block (the block's first key plus 0.05
    # N(0,1)): rows select some blocks and the zeroth-order term of the others
    # carries a large share of the output (about half or more on these inputs,
    # against ~1e-6 on the Fourier-feature workloads), so a slip in the
    # approximation path fails here (method: proxy-score reuse, Eq. 8-10).
    wl = WORKLOADS[shape]
    qb, kb, vb = fourier_inputs(wl)
    kb = near_block_constant_keys(kb, 0.05, seed=71)
    out, sel, _ = _full_check(qb, kb, vb, beta, wl.chunk, mask_heads=range(wl.B * wl.H))
    n_sel = sel.sum(axis=-1)
    assert ((n_sel > 0) & (n_sel < wl.N)).any()        # mixed rows exist
    exact, _, _ = run_gpu(qb, kb, vb, beta, wl.chunk, flags=sa.FLAG_EXACT_ONLY, debug=False)
    assert np.linalg.norm(out - exact) > 0.1 * np.linalg.norm(out)


@pytest.mark.parametrize("L,d,chunk", [(1, 128, 4), (64, 128, 1), (65, 64, 2), (127, 128, 4), (129, 64, 3),
                                       (1000, 128, 5), (4033, 64, 16), (4096, 128, 200)])
@pytest.mark.parametrize("beta", [0.75, -math.inf, math.inf])
def test_edge_shapes(L, d, chunk, beta):
    qb, kb, vb = custom_fourier(2, 2, (1, 1, L), d, 2.0, seed=L * 7 + d)
    _full_check(qb, kb, vb, beta, chunk)


def test_maximum_length_sampled():
    # The longest sequence accepted: L = 2^20, N = 16384 pooled blocks, 512 mask
    # words per row; one head, sampled query blocks including the first and last.
    qb, kb, vb = gauss_inputs(1, 1, 1 << 20, 64, seed=17)
    _full_check(qb, kb, vb, 1.5, 64, rows=[0, 1, 5000, 12345, 16382, 16383])


def test_gaussian_inputs_density():
    qb, kb, vb = gauss_inputs(1, 2, 64 * 512, 128, seed=12)
    for beta, rho in ((0.5, 0.3085), (1.0, 0.1587), (1.5, 0.0668)):
        out, sel, rep = _full_check(qb, kb, vb, beta, 64, rows=list(range(0, 512, 37)) + [511])
        _, _, counts = run_gpu(qb, kb, vb, beta, 64, debug=False)
        assert abs(counts.mean() / 512 - rho) < 0.01


def test_host_buffer_entry_point_matches_device_call():
    wl = WORKLOADS["small"]
    qb, kb, vb = fourier_inputs(wl)
    dev, _, _ = run_gpu(qb, kb, vb, 1.0, wl.chunk, debug=False)
    host = sa.forward_host(qb, kb, vb, 1.0, wl.chunk, flags=sa.FLAG_SYNC_CHECK)
    import torch
    got = torch.from_numpy(host.view(np.int16)).view(torch.bfloat16).float().numpy()
    assert np.array_equal(got, dev)


def test_host_buffer_entry_point_in_groups():
    # 9 (batch, head) slices go through in 5 groups of 2, 2, 2, 2 and 1: the
    # result equals one device call on all of them, bit for bit
    import torch
    qb, kb, vb = gauss_inputs(3, 3, 1000, 64, seed=77)
    dev, _, _ = run_gpu(qb, kb, vb, 0.75, 5, debug=False)
    host = sa.forward_host(qb, kb, vb, 0.75, 5, flags=sa.FLAG_SYNC_CHECK)
    got = torch.from_numpy(host.view(np.int16)).view(torch.bfloat16).float().numpy()
    assert np.array_equal(got, dev)


def test_staged_calls_match_forward():
    import torch
    from parity_util import to_device
    wl = WORKLOADS["small"]
    qb, kb, vb = fourier_inputs(wl)
    ref, _, _ = run_gpu(qb, kb, vb, 1.0, wl.chunk, debug=False)
    q, k, v = to_device(qb), to_device(kb), to_device(vb)
    out = torch.empty_like(q)
    sa.stage_pool(q, k, v)
    sa.stage_threshold(wl.B, wl.H, wl.L, wl.d, 1.0)
    sa.stage_fused(q, k, v, out, wl.chunk, flags=sa.FLAG_SYNC_CHECK)
    torch.cuda.synchronize()
    assert np.array_equal(out.float().cpu().numpy(), ref)


def test_runtime_errors_on_device():
    import torch
    from parity_util import to_device
    wl = WORKLOADS["tiny"]
    qb, kb, vb = fourier_inputs(wl)
    q, k, v = to_device(qb), to_device(kb), to_device(vb)
    flat = torch.empty(q.numel() + 8, dtype=torch.bfloat16, device="cuda")
    mis = flat[1:1 + q.numel()].view(q.shape)       # 2-byte offset: misaligned
    with pytest.raises(sa.SolAttnError) as e:
        sa.forward(mis, k, v, 1.0, 4)
    assert e.value.code == -3
    sa.forward(q, k, v, 1.0, 4)
    with pytest.raises(sa.SolAttnError) as e:
        sa.stats(1, 1, 2048)                          # no forward of that shape
    assert e.value.code == -6
    with pytest.raises(sa.SolAttnError) as e:
        sa.stage_fused(q, k, v, torch.empty_like(q), 4) if False else sa.stage_threshold(1, 3, 1024, 64, 1.0)
    assert e.value.code == -6


@pytest.mark.parametrize("beta", [0.75, 1.0, 1.5])
def test_approximation_ablation_on_device(beta):
    # method: the zeroth-order term is exact when every key of a block equals the
    # block's mean, so there the full method reproduces select-all attention for
    # any beta while exact-only (no approximation of unselected blocks, same
    # selection) does not; experiments, ablation of the approximation
    import torch
    wl = WORKLOADS["small"]
    qb, kb, vb = fourier_inputs(wl)
    kb = kb.copy()
    B, H, L, d = kb.shape
    for j in range(0, L, 64):   # every key of block j := the block's first key
        kb[:, :, j:j + 64, :] = kb[:, :, j:j + 1, :]
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    q, k, v = dev(qb), dev(kb), dev(vb)
    dense = sa.forward(q, k, v, -math.inf, wl.chunk, flags=sa.FLAG_SELECT_ALL).float()
    full = sa.forward(q, k, v, beta, wl.chunk).float()
    exact = sa.forward(q, k, v, beta, wl.chunk, flags=sa.FLAG_EXACT_ONLY).float()
    rel = lambda o: (torch.linalg.vector_norm(o - dense) / torch.linalg.vector_norm(dense)).item()
    r_full, r_exact = rel(full), rel(exact)
    print(f"beta={beta} rel-l2 vs select-all: approx {r_full:.2e} exact-only {r_exact:.2e}")
    assert r_full < 5e-3              # bf16 rounding of P and of the output only
    assert r_exact > 10 * max(r_full, 1e-4)


def test_bounded_wait_runs_out_and_the_next_forward_is_clean():
    # Failure path of the fused kernel's bounded waits: with the test-stall flag
    # its routing step publishes no work, every waiting role gives up after
    # 1 ms and leaves, TMEM is released and the status word says "timeout".
    # The context stays usable: the next forward (status cleared) passes parity.
    import torch
    from parity_util import to_device
    wl = WORKLOADS["tiny"]
    qb, kb, vb = fourier_inputs(wl)
    q, k, v = to_device(qb), to_device(kb), to_device(vb)
    with pytest.raises(sa.SolAttnError) as e:
        sa.forward(q, k, v, 1.0, wl.chunk, flags=sa.FLAG_TEST_STALL | sa.FLAG_SYNC_CHECK)
    assert e.value.code == -5
    assert "timed out" in str(e.value)
    torch.cuda.synchronize()
    _full_check(qb, kb, vb, 1.0, wl.chunk)


@pytest.mark.parametrize("beta", [0.75, 1.0, 1.5, math.inf])
@pytest.mark.parametrize("case", ["tiny", "small", "small_blocky", "ragged"])
def test_first_order_flag(case, beta):
    # Extension of the proxy-score reuse (Eq. 8): unselected blocks take the
    # first-order expansion around their row-wise mean score; against the
    # oracle's taylor_order=1 on identical inputs.
    if case == "ragged":
        qb, kb, vb = custom_fourier(1, 2, (1, 1, 1000), 128, 2.0, seed=401)
        chunk = 5
    else:
        wl = WORKLOADS["tiny" if case == "tiny" else "small"]
        qb, kb, vb = fourier_inputs(wl)
        chunk = wl.chunk
        if case == "small_blocky":
            kb = near_block_constant_keys(kb, 0.1, seed=73)
    _full_check(qb, kb, vb, beta, chunk, flags=sa.FLAG_FIRST_ORDER)


def test_first_order_is_closer_to_dense_on_near_constant_keys():
    # With keys K̄_j + eps R the zeroth-order error is O(eps), the first-order O(eps^2)
    wl = WORKLOADS["small"]
    qb, kb, vb = fourier_inputs(wl)
    kb = near_block_constant_keys(kb, 0.1, seed=73)
    dense, _, _ = run_gpu(qb, kb, vb, -math.inf, wl.chunk, debug=False)
    zero, _, _ = run_gpu(qb, kb, vb, 1.0, wl.chunk, debug=False)
    first, _, _ = run_gpu(qb, kb, vb, 1.0, wl.chunk, flags=sa.FLAG_FIRST_ORDER, debug=False)
    e0 = np.linalg.norm(zero - dense) / np.linalg.norm(dense)
    e1 = np.linalg.norm(first - dense) / np.linalg.norm(dense)
    print(f"rel-l2 vs select-all: zeroth order {e0:.2e}, first order {e1:.2e}")
    assert e1 < 0.5 * e0


def test_conflicting_flags_are_rejected():
    from parity_util import to_device
    wl = WORKLOADS["tiny"]
    q, k, v = (to_device(x) for x in fourier_inputs(wl))
    with pytest.raises(sa.SolAttnError) as e:
        sa.forward(q, k, v, 1.0, wl.chunk, flags=sa.FLAG_FIRST_ORDER | sa.FLAG_EXACT_ONLY)
    assert e.value.code == -1


@pytest.mark.parametrize("kk", [0, 1, 13, 64])
def test_topk_comparison_router(kk):
    # The comparison router of the routing-cost report (experiments: top-k
    # routing over the materialised proxy map, Fig. 5b): each row keeps exactly
    # min(k, N) blocks, and every kept block's oracle proxy logit is at least
    # every dropped one's (up to fp32 rounding of the map, 1e-4).
    import torch
    from oracle import pool_blocks, proxy_logits
    from parity_util import to_device
    from synth import bf16_bits_to_f64
    wl = WORKLOADS["small"]
    qb, kb, vb = fourier_inputs(wl)
    q, k, v = to_device(qb), to_device(kb), to_device(vb)
    sa.stage_pool(q, k, v)
    mask = sa.topk_route(wl.B, wl.H, wl.L, wl.d, kk)
    torch.cuda.synchronize()
    w = mask.to(torch.int64).cpu().numpy() & 0xFFFFFFFF
    N = wl.N
    sel = ((w[..., :, None] >> np.arange(32)) & 1).reshape(wl.B, wl.H, N, -1)[..., :N].astype(bool)
    for h in range(wl.H):
        qbar, _, _ = pool_blocks(bf16_bits_to_f64(qb[0, h]))
        kbar, _, _ = pool_blocks(bf16_bits_to_f64(kb[0, h]))
        s = proxy_logits(qbar, kbar)
        for i in range(N):
            row = sel[0, h, i]
            assert row.sum() == min(kk, N)
            if 0 < kk < N:
                assert s[i][row].min() >= s[i][~row].max() - 1e-4
