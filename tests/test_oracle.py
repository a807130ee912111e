"""Pins of the fp64 oracle against facts the pages and the mathematics fix.

Each pin is independent of the oracle's own code path: hand-derived golden masks,
library routines (torch float64 softmax / scaled_dot_product_attention,
numpy.linalg.norm), special cases where the piecewise form is exact, the
whole-head identity for H-bar, brute-force subset search for routing and the Taylor
error order. A plausible slip in the oracle (a dropped term, a missing scale, a
transposed H, a wrong sign, a sum for a mean) fails at least one of them.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _read_rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


# ------------------------------------------------------------------------- mask
def test_mask_page1_example_matches_hand_derivation():
    # 77 text tokens -> 1 block of 128; 1024 image tokens -> 8 blocks on a 1 x 8 grid;
    # window 2, global stride 4 ("多模态 DiT 上的块稀疏 Attention" §4.2).
    keep = orc.mask_dense(1, 1, 8, 2, 4)
    want = np.array([[int(c) for c in r[0]] for r in _read_rows(
        "page1_mask_T77_I1024_B128.txt")], dtype=bool)
    assert keep.shape == (9, 9)
    assert (keep == want).all()
    assert keep.sum() == 59


def test_mask_multimodal_dit_row_lengths():
    keep = orc.mask_dense(2, 4, 4, 1, 16)
    rows = [int(x) for r in _read_rows("multimodal_dit_row_lengths.txt") for x in r]
    assert keep.sum(axis=1).tolist() == rows
    assert keep.sum() == 180 and keep.size == 324


def test_mask_large_radius_is_full_and_rows_full_option():
    assert orc.mask_dense(3, 4, 5, 10, 7).all()
    # global_rows_full: global image blocks 0 and 4 of a 1x8 grid get full rows
    keep = orc.mask_dense(1, 1, 8, 0, 4, global_rows_full=1)
    assert keep[1].all() and keep[5].all()
    assert keep[2].sum() == 1 + 1 + 2      # text + itself + globals 0 and 4


def test_csr_roundtrip():
    keep = orc.mask_dense(2, 4, 4, 1, 16)
    rp, ci = orc.dense_to_csr(keep)
    assert rp[-1] == 180
    back = np.zeros_like(keep)
    for i in range(keep.shape[0]):
        seg = ci[rp[i]:rp[i + 1]]
        assert (np.diff(seg) > 0).all()
        back[i, seg] = True
    assert (back == keep).all()


# ------------------------------------------------------------- keep-or-drop / dense
def _torch_masked_softmax_attention(q, k, v, keep_tok, scale):
    """Textbook masked attention: -inf on dropped keys, library softmax."""
    qt, kt, vt = (torch.from_numpy(np.asarray(x, dtype=np.float64)) for x in (q, k, v))
    a = scale * qt @ kt.T
    a = a.masked_fill(~torch.from_numpy(keep_tok), float("-inf"))
    return (torch.softmax(a, dim=-1) @ vt).numpy(), torch.logsumexp(a, dim=-1).numpy()


@pytest.mark.parametrize("block,M,d", [(8, 6, 16), (16, 5, 32)])
def test_keep_or_drop_equals_masked_softmax(block, M, d):
    r = _rng(1)
    L = block * M
    q, k, v = r.standard_normal((3, L, d))
    keep = r.random((M, M)) < 0.5
    keep[np.arange(M), np.arange(M)] = True
    rp, ci = orc.dense_to_csr(keep)
    scale = 1 / math.sqrt(d)
    out, lse = orc.keep_or_drop_head(q, k, v, rp, ci, block, scale)
    keep_tok = np.kron(keep, np.ones((block, block), dtype=bool))
    ref, ref_lse = _torch_masked_softmax_attention(q, k, v, keep_tok, scale)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def _sdpa(q, k, v, scale):
    qt, kt, vt = (torch.from_numpy(np.asarray(x, dtype=np.float64))[None, None]
                  for x in (q, k, v))
    return torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, scale=scale)[0, 0].numpy()


def test_dense_head_equals_sdpa():
    r = _rng(2)
    q, k, v = r.standard_normal((3, 40, 24))
    np.testing.assert_allclose(orc.dense_head(q, k, v, 0.3), _sdpa(q, k, v, 0.3),
                               rtol=1e-12, atol=1e-12)


def test_full_density_keep_or_drop_and_pisa_equal_dense():
    r = _rng(3)
    block, M, d = 8, 5, 16
    L = block * M
    q, k, v = r.standard_normal((3, L, d))
    scale = 1 / math.sqrt(d)
    rp, ci = orc.dense_to_csr(np.ones((M, M), dtype=bool))
    kbar, vsum, H, Hbar, Mn = orc.precompute_head(k, v, block)
    ref = _sdpa(q, k, v, scale)
    kod, _ = orc.keep_or_drop_head(q, k, v, rp, ci, block, scale)
    pisa, _ = orc.pisa_head(q, k, v, rp, ci, block, scale, kbar, vsum, Hbar)
    np.testing.assert_allclose(kod, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(pisa, ref, rtol=1e-12, atol=1e-12)


def test_keep_or_drop_is_dense_renormalised_over_selected_blocks():
    # Keep-or-drop = dense attention weights restricted to S_i and renormalised.
    r = _rng(4)
    block, M, d = 4, 6, 8
    L = block * M
    q, k, v = r.standard_normal((3, L, d))
    scale = 0.5
    keep = r.random((M, M)) < 0.4
    keep[:, 0] = True
    rp, ci = orc.dense_to_csr(keep)
    out, _ = orc.keep_or_drop_head(q, k, v, rp, ci, block, scale)
    w = np.exp(scale * q @ k.T)
    w /= w.sum(axis=1, keepdims=True)                 # dense weights
    w *= np.kron(keep, np.ones((block, block)))
    w /= w.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(out, w @ v, rtol=1e-11, atol=1e-12)


def test_keep_or_drop_empty_row_outputs_zero():
    q, k, v = _rng(5).standard_normal((3, 8, 4))
    rp = np.array([0, 0, 2], dtype=np.int32)
    ci = np.array([0, 1], dtype=np.int32)
    out, lse = orc.keep_or_drop_head(q, k, v, rp, ci, 4, 0.5)
    assert (out[:4] == 0).all() and np.isneginf(lse[:4]).all()


# ------------------------------------------------------------------- precompute
def test_precompute_whole_head_identities():
    r = _rng(6)
    block, M, d = 8, 7, 6
    k = r.standard_normal((block * M, d)) + 2.0
    v = r.standard_normal((block * M, d)) - 1.0
    kbar, vsum, H, Hbar, Mn = orc.precompute_head(k, v, block)
    # kbar is the MEAN, vsum the SUM of the block (B * kbar = block sum)
    np.testing.assert_allclose(block * kbar, k.reshape(M, block, d).sum(1), rtol=1e-13)
    np.testing.assert_allclose(vsum.sum(0), v.sum(0), rtol=1e-12, atol=1e-12)
    # whole-head, uncentred identity: M Hbar = K^T V - sum_j kbar_j^T vsum_j
    np.testing.assert_allclose(M * Hbar, k.T @ v - kbar.T @ vsum, rtol=1e-11, atol=1e-11)
    # H_j orientation: d_k rows, d_v cols (q_t H is a row in value space)
    j = 3
    kb, vb = k[j * block:(j + 1) * block], v[j * block:(j + 1) * block]
    np.testing.assert_allclose(H[j], kb.T @ vb - np.outer(kbar[j], vsum[j]), atol=1e-11)
    for jj in range(M):
        assert Mn[jj] == pytest.approx(np.linalg.norm(H[jj] - Hbar, "fro"), rel=1e-13)


def test_first_order_term_adds_nothing_to_denominator():
    # sum_n (k_{j,n} - kbar_j) = 0: the first-order Taylor term of the denominator
    # sum_n alpha (1 + s q (k_n - kbar)) equals B alpha exactly.
    r = _rng(7)
    block, M, d = 16, 4, 8
    k = 3.0 * r.standard_normal((block * M, d)) + 5.0
    v = r.standard_normal((block * M, d))
    kbar, *_ = orc.precompute_head(k, v, block)
    resid = (k.reshape(M, block, d) - kbar[:, None]).sum(axis=1)
    assert np.abs(resid).max() <= 1e-12 * np.abs(k).max() * block
    q = r.standard_normal(d)
    for j in range(M):
        alpha = math.exp(0.3 * q @ kbar[j])
        first = sum(alpha * (1 + 0.3 * q @ (k[j * block + n] - kbar[j]))
                    for n in range(block))
        assert first == pytest.approx(block * alpha, rel=1e-12)


# ------------------------------------------------------------------- PISA exactness
def _random_csr(M, kk, seed):
    r = _rng(seed)
    keep = np.zeros((M, M), dtype=bool)
    for i in range(M):
        keep[i, r.choice(M, size=kk, replace=False)] = True
    return orc.dense_to_csr(keep)


def test_pisa_block_size_one_is_exact():
    r = _rng(8)
    L, d = 24, 8
    q, k, v = r.standard_normal((3, L, d))
    scale = 1 / math.sqrt(d)
    kbar, vsum, H, Hbar, _ = orc.precompute_head(k, v, 1)
    assert np.abs(H).max() == 0 and np.abs(Hbar).max() == 0
    rp, ci = _random_csr(L, 5, 9)
    out, _ = orc.pisa_head(q, k, v, rp, ci, 1, scale, kbar, vsum, Hbar)
    np.testing.assert_allclose(out, _sdpa(q, k, v, scale), rtol=1e-12, atol=1e-12)


def test_pisa_constant_key_blocks_are_exact():
    r = _rng(10)
    block, M, d = 8, 6, 16
    centres = r.standard_normal((M, d))
    k = np.repeat(centres, block, axis=0)
    q, v = r.standard_normal((2, block * M, d))
    scale = 1 / math.sqrt(d)
    kbar, vsum, H, Hbar, _ = orc.precompute_head(k, v, block)
    assert np.abs(Hbar).max() < 1e-12
    rp, ci = _random_csr(M, 2, 11)
    out, _ = orc.pisa_head(q, k, v, rp, ci, block, scale, kbar, vsum, Hbar)
    np.testing.assert_allclose(out, _sdpa(q, k, v, scale), rtol=1e-11, atol=1e-12)


def test_pisa_lse_is_log_denominator():
    r = _rng(12)
    block, M, d = 8, 5, 8
    q, k, v = r.standard_normal((3, block * M, d))
    kbar, vsum, H, Hbar, _ = orc.precompute_head(k, v, block)
    rp, ci = _random_csr(M, 2, 13)
    scale = 0.4
    out, lse = orc.pisa_head(q, k, v, rp, ci, block, scale, kbar, vsum, Hbar, qblocks=[2])
    sel = set(ci[rp[2]:rp[3]].tolist())
    qi = q[2 * block:3 * block]
    den = np.zeros(block)
    for j in range(M):
        if j in sel:
            den += np.exp(scale * qi @ k[j * block:(j + 1) * block].T).sum(1)
        else:
            den += block * np.exp(scale * qi @ kbar[j])
    np.testing.assert_allclose(lse, np.log(den), rtol=1e-12)


def _taylor_errors(eps_list, same_cov):
    """Max error vs dense for zeroth-order, per-block first-order and global-Hbar
    PISA when K_j = c_j + eps * N_j."""
    r = _rng(14)
    block, M, d = 16, 6, 8
    scale = 1 / math.sqrt(d)
    q = r.standard_normal((block * M, d))
    c = r.standard_normal((M, 1, d))
    if same_cov:
        noise = np.broadcast_to(r.standard_normal((1, block, d)), (M, block, d))
        v = np.tile(r.standard_normal((block, d)), (M, 1))
    else:
        noise = r.standard_normal((M, block, d))
        v = r.standard_normal((block * M, d))
    rp, ci = _random_csr(M, 2, 15)
    errs = {"zeroth": [], "perblock": [], "global": []}
    for eps in eps_list:
        k = (c + eps * noise).reshape(block * M, d)
        kbar, vsum, H, Hbar, _ = orc.precompute_head(k, v, block)
        ref = _sdpa(q, k, v, scale)
        z, _ = orc.zeroth_order_head(q, k, v, rp, ci, block, scale, kbar, vsum)
        p, _ = orc.pisa_head(q, k, v, rp, ci, block, scale, kbar, vsum, Hbar, Hblocks=H)
        g, _ = orc.pisa_head(q, k, v, rp, ci, block, scale, kbar, vsum, Hbar)
        errs["zeroth"].append(np.abs(z - ref).max())
        errs["perblock"].append(np.abs(p - ref).max())
        errs["global"].append(np.abs(g - ref).max())
    return errs


def _slope(eps, err):
    return np.polyfit(np.log(eps), np.log(err), 1)[0]


def test_taylor_error_orders():
    eps = [0.005, 0.01, 0.02, 0.04]
    e = _taylor_errors(eps, same_cov=False)
    assert 0.85 < _slope(eps, e["zeroth"]) < 1.15
    assert 1.85 < _slope(eps, e["perblock"]) < 2.15
    assert 0.85 < _slope(eps, e["global"]) < 1.15
    # identical per-block covariance: Hbar == H_j, so the global correction is the
    # exact first-order term and the error drops to second order
    e2 = _taylor_errors(eps, same_cov=True)
    assert 1.85 < _slope(eps, e2["global"]) < 2.15
    assert e2["global"][0] < 0.05 * e2["zeroth"][0]


# ---------------------------------------------------------------------- routing
def test_route_lambda_zero_is_topk_of_pooled_scores():
    r = _rng(16)
    block, M, d = 4, 9, 8
    q = r.standard_normal((block * M, d))
    kbar = r.standard_normal((M, d))
    Mn = r.random(M)
    rp, ci, sc = orc.route_head(q, kbar, Mn, block, 3, 0.0, 0.35)
    raw = q.reshape(M, block, d).sum(1) @ kbar.T     # monotone in the pooled score
    np.testing.assert_allclose(sc.sum(axis=1), 1.0, rtol=1e-13)
    for i in range(M):
        want = np.sort(np.argsort(-raw[i], kind="stable")[:3])
        assert ci[3 * i:3 * i + 3].tolist() == want.tolist()


def test_route_brute_force_subset_maximises_score():
    r = _rng(17)
    block, M, d = 4, 7, 5
    q = r.standard_normal((block * M, d))
    kbar = r.standard_normal((M, d))
    Mn = r.random(M) * 3
    lam, kk, scale = 0.7, 3, 0.5
    rp, ci, _ = orc.route_head(q, kbar, Mn, block, kk, lam, scale)
    qbar = q.reshape(M, block, d).mean(1)
    for i in range(M):
        a = scale * qbar[i] @ kbar.T
        p = np.exp(a) / np.exp(a).sum()
        s = p + lam * Mn / Mn.sum()
        best = max(itertools.combinations(range(M), kk), key=lambda c: s[list(c)].sum())
        assert ci[kk * i:kk * (i + 1)].tolist() == list(best)


def test_route_large_lambda_follows_covariance_norm_and_ties_go_low():
    r = _rng(18)
    block, M, d = 4, 8, 6
    q = r.standard_normal((block * M, d))
    kbar = r.standard_normal((M, d))
    Mn = np.array([1.0, 5.0, 2.0, 5.0, 0.5, 4.0, 3.0, 0.1])
    rp, ci, _ = orc.route_head(q, kbar, Mn, block, 3, 1e6, 0.3)
    for i in range(M):
        assert ci[3 * i:3 * i + 3].tolist() == [1, 3, 5]
    # exact ties: identical centroids and lambda 0 -> the smaller index wins
    kbar2 = np.zeros((M, d))
    rp, ci, _ = orc.route_head(q, kbar2, Mn, block, 2, 0.0, 0.3)
    for i in range(M):
        assert ci[2 * i:2 * i + 2].tolist() == [0, 1]
    # all-equal covariance norms contribute a constant: same as lambda 0
    _, c1, _ = orc.route_head(q, kbar, np.ones(M), block, 3, 5.0, 0.3)
    _, c0, _ = orc.route_head(q, kbar, np.ones(M), block, 3, 0.0, 0.3)
    assert c1.tolist() == c0.tolist()


def test_batched_route_csr_layout():
    r = _rng(19)
    BH, block, M, d = 3, 4, 5, 4
    q = r.standard_normal((BH, block * M, d))
    kbar = r.standard_normal((BH, M, d))
    Mn = r.random((BH, M))
    rp, ci, sc = orc.route(q, kbar, Mn, block, 2, 1.0, 0.5)
    assert rp.shape == (BH * (M + 1),) and ci.shape == (BH * M * 2,)
    for h in range(BH):
        hrp, hci = orc.head_csr(rp, ci, h, M, True)
        rp1, ci1, _ = orc.route_head(q[h], kbar[h], Mn[h], block, 2, 1.0, 0.5)
        assert hrp.tolist() == rp1.tolist() and hci.tolist() == ci1.tolist()


# ------------------------------------------------------------- token-level padding
def _padded_case(seed, M=6, block=8, d=8):
    """A head whose blocks 0 and 3 carry padding at their tail (a text segment padded
    to the block size, and a one-token timestep block)."""
    r = _rng(seed)
    q, k, v = r.standard_normal((3, M * block, d))
    valid = [block] * M
    valid[0], valid[3] = 5, 1
    return q, k, v, valid, block


def _garbage(x, valid, block, seed):
    """The same tensor with every padded row replaced by large random values."""
    y = np.array(x, copy=True)
    r = _rng(seed)
    for j, n in enumerate(valid):
        y[j * block + n:(j + 1) * block] = 1e3 * r.standard_normal((block - n, y.shape[1]))
    return y


def _masked_sdpa(q, k, v, scale, allowed):
    """torch float64 scaled_dot_product_attention with a boolean key mask."""
    qt, kt, vt = (torch.from_numpy(np.asarray(x, dtype=np.float64))[None, None]
                  for x in (q, k, v))
    m = torch.from_numpy(allowed)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m,
                                                            scale=scale)[0, 0].numpy()


def test_padding_with_full_blocks_changes_nothing():
    q, k, v, _, block = _padded_case(20)
    M = q.shape[0] // block
    full = [block] * M
    s = 1 / math.sqrt(q.shape[1])
    rp, ci = _random_csr(M, 3, 21)
    a = orc.precompute_head(k, v, block)
    b_ = orc.precompute_head(k, v, block, key_valid=full)
    for x, y in zip(a, b_):
        np.testing.assert_array_equal(x, y)
    np.testing.assert_array_equal(orc.keep_or_drop_head(q, k, v, rp, ci, block, s)[0],
                                  orc.keep_or_drop_head(q, k, v, rp, ci, block, s, key_valid=full)[0])
    kbar, vsum, H, Hbar, Mn = a
    np.testing.assert_array_equal(
        orc.pisa_head(q, k, v, rp, ci, block, s, kbar, vsum, Hbar)[0],
        orc.pisa_head(q, k, v, rp, ci, block, s, kbar, vsum, Hbar, key_valid=full)[0])
    np.testing.assert_array_equal(orc.route_head(q, kbar, Mn, block, 2, 1.0, s)[1],
                                  orc.route_head(q, kbar, Mn, block, 2, 1.0, s, key_valid=full)[1])


def test_padded_rows_do_not_matter():
    """Nothing computed for real tokens depends on what the padded positions hold."""
    q, k, v, valid, block = _padded_case(22)
    M = q.shape[0] // block
    s = 1 / math.sqrt(q.shape[1])
    q2, k2, v2 = (_garbage(x, valid, block, 23 + n) for n, x in enumerate((q, k, v)))
    st1 = orc.precompute_head(k, v, block, key_valid=valid)
    st2 = orc.precompute_head(k2, v2, block, key_valid=valid)
    for x, y in zip(st1, st2):
        np.testing.assert_allclose(x, y, rtol=1e-12, atol=1e-12)
    kbar, vsum, H, Hbar, Mn = st1
    rp1, ci1, sc1 = orc.route_head(q, kbar, Mn, block, 3, 1.0, s, key_valid=valid)
    rp2, ci2, sc2 = orc.route_head(q2, kbar, Mn, block, 3, 1.0, s, key_valid=valid)
    np.testing.assert_array_equal(ci1, ci2)
    np.testing.assert_allclose(sc1, sc2, rtol=1e-12, atol=1e-12)
    real = np.concatenate([np.arange(j * block, j * block + valid[j]) for j in range(M)])
    o1, _ = orc.pisa_head(q, k, v, rp1, ci1, block, s, kbar, vsum, Hbar, key_valid=valid)
    o2, _ = orc.pisa_head(q2, k2, v2, rp1, ci1, block, s, kbar, vsum, Hbar, key_valid=valid)
    np.testing.assert_allclose(o1[real], o2[real], rtol=1e-12, atol=1e-12)
    o1, _ = orc.keep_or_drop_head(q, k, v, rp1, ci1, block, s, key_valid=valid)
    o2, _ = orc.keep_or_drop_head(q2, k2, v2, rp1, ci1, block, s, key_valid=valid)
    np.testing.assert_allclose(o1[real], o2[real], rtol=1e-12, atol=1e-12)


def test_keep_or_drop_with_padding_is_masked_sdpa():
    q, k, v, valid, block = _padded_case(24)
    M = q.shape[0] // block
    s = 1 / math.sqrt(q.shape[1])
    rp, ci = _random_csr(M, 3, 25)
    out, _ = orc.keep_or_drop_head(q, k, v, rp, ci, block, s, key_valid=valid)
    allowed = np.zeros((q.shape[0], q.shape[0]), dtype=bool)
    for i in range(M):
        for j in ci[rp[i]:rp[i + 1]]:
            allowed[i * block:(i + 1) * block, j * block:j * block + valid[j]] = True
    np.testing.assert_allclose(out, _masked_sdpa(q, k, v, s, allowed), rtol=1e-10, atol=1e-12)


def test_pisa_full_selection_with_padding_is_masked_dense():
    q, k, v, valid, block = _padded_case(26)
    M = q.shape[0] // block
    s = 1 / math.sqrt(q.shape[1])
    rp, ci = orc.dense_to_csr(np.ones((M, M), dtype=bool))
    kbar, vsum, H, Hbar, Mn = orc.precompute_head(k, v, block, key_valid=valid)
    out, lse = orc.pisa_head(q, k, v, rp, ci, block, s, kbar, vsum, Hbar, key_valid=valid)
    allowed = np.zeros((q.shape[0], q.shape[0]), dtype=bool)
    for j in range(M):
        allowed[:, j * block:j * block + valid[j]] = True
    np.testing.assert_allclose(out, _masked_sdpa(q, k, v, s, allowed), rtol=1e-10, atol=1e-12)


def test_padded_block_statistics_use_real_tokens_only():
    """A block whose real keys are all one vector c (padding holds other values) has
    centroid c and H_j = 0; its value sum counts the real rows only."""
    q, k, v, valid, block = _padded_case(27)
    c = _rng(28).standard_normal(k.shape[1])
    k = np.array(k, copy=True)
    k[0:valid[0]] = c
    kbar, vsum, H, Hbar, Mn = orc.precompute_head(k, v, block, key_valid=valid)
    np.testing.assert_allclose(kbar[0], c, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(H[0], 0.0, atol=1e-12)
    np.testing.assert_allclose(vsum[0], np.asarray(v)[0:valid[0]].sum(axis=0), rtol=1e-13)
    np.testing.assert_allclose(kbar[3], k[3 * block], rtol=1e-13)   # the one-token block


def test_routing_places_every_padded_block_in_every_list():
    q, k, v, valid, block = _padded_case(29)
    M = q.shape[0] // block
    s = 1 / math.sqrt(q.shape[1])
    kbar, vsum, H, Hbar, Mn = orc.precompute_head(k, v, block, key_valid=valid)
    for kk in (2, 4):
        rp, ci, sc = orc.route_head(q, kbar, Mn, block, kk, 1.0, s, key_valid=valid)
        for i in range(M):
            row = list(ci[rp[i]:rp[i + 1]])
            assert 0 in row and 3 in row and row == sorted(row) and len(row) == kk
    with pytest.raises(ValueError):
        orc.route_head(q, kbar, Mn, block, 1, 1.0, s, key_valid=valid)


def test_pisa_padded_block_in_the_tail_weighs_its_real_tokens():
    """A padded block left in U_i (the oracle accepts such lists; the GPU refuses them).
    When every block's real keys are one vector c_j, the zeroth-order term of block j
    is exact: sum over its real keys of e^{s q.c_j} v_n = alpha_tj vsum_j and the
    denominator gains (real tokens) x alpha_tj, while H_j = 0 and Hbar = 0. PISA then
    equals softmax attention over the real keys only, whatever the lists; a tail
    weight of B instead of the real-token count, or pad rows in the value sum, breaks
    the equality."""
    q, k, v, valid, block = _padded_case(30)
    M = q.shape[0] // block
    s = 1 / math.sqrt(q.shape[1])
    centres = _rng(31).standard_normal((M, k.shape[1]))
    k = np.array(k, copy=True)
    for j in range(M):
        k[j * block:j * block + valid[j]] = centres[j]
    k, v = (_garbage(x, valid, block, 32 + n) for n, x in enumerate((k, v)))
    kbar, vsum, H, Hbar, Mn = orc.precompute_head(k, v, block, key_valid=valid)
    assert np.abs(Hbar).max() < 1e-12
    # lists that leave both padded blocks (0 and 3) out of some rows
    keep = np.zeros((M, M), dtype=bool)
    keep[:, 1] = True
    keep[0, 0] = keep[2, 3] = keep[4, 5] = True
    rp, ci = orc.dense_to_csr(keep)
    assert any(0 not in ci[rp[i]:rp[i + 1]] for i in range(M))
    assert any(3 not in ci[rp[i]:rp[i + 1]] for i in range(M))
    out, lse = orc.pisa_head(q, k, v, rp, ci, block, s, kbar, vsum, Hbar, key_valid=valid)
    allowed = np.zeros((q.shape[0], q.shape[0]), dtype=bool)
    for j in range(M):
        allowed[:, j * block:j * block + valid[j]] = True
    np.testing.assert_allclose(out, _masked_sdpa(q, k, v, s, allowed), rtol=1e-10, atol=1e-12)
