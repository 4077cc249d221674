"""Pins for the CPU oracle: each test ties one part of the oracle to something other than
the oracle itself -- a figure the RAM-Net project page prints, a closed form, a library
routine, a special case that reduces to a textbook result, or brute force on tiny inputs.

Page cited throughout: "RAM-Net: Linear-Time Sequence Modeling with Sparsely Addressable
State", project page (muoncat.github.io/ramnet_web); paragraphs named in each test.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import OracleConfig

RNG = np.random.default_rng(1234)


def _digits(i, d_p, U):
    # big-endian digits of slot i (numpy's C-order unravel: first axis most significant)
    return np.array(np.unravel_index(i, (d_p,) * U)).T


def _summed_logits(x, d_p, U):
    """s_i = sum_u x_u[d_u(i)] for all M slots, built with numpy's mixed-radix unravel."""
    M = d_p ** U
    dig = _digits(np.arange(M), d_p, U)                 # [M, U]
    xs = x.reshape(U, d_p)
    return xs[np.arange(U)[None, :], dig].sum(axis=1)   # [M]


def _read_facts(golden_dir):
    facts = []
    with open(os.path.join(golden_dir, "pages_facts.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            kind, *kv = line.split()
            facts.append((kind, dict(p.split("=") for p in kv)))
    return facts


# ------------------------------------------------------------------ Product Softmax

def test_page_example_1024_slots_from_20_scores(golden_dir):
    """Product Softmax paragraph: M = 4^5 = 1024 slots from 20 scores; every slot is
    reachable and the full product distribution sums to one."""
    (kind, f), = [x for x in _read_facts(golden_dir) if x[0] == "product_softmax"]
    cfg = OracleConfig(d_p=int(f["d_p"]), U=int(f["U"]), K=int(f["M"]), d_v=1)
    assert cfg.M == int(f["M"]) and cfg.L == int(f["scores"])
    x = RNG.normal(0, 1.5, cfg.L)
    idx, _ = oracle.topk_bruteforce(x, cfg.d_p, cfg.U, cfg.M)
    assert sorted(idx.tolist()) == list(range(cfg.M))
    w = oracle.weights(x, cfg.d_p, cfg.U, idx, renorm=0)
    assert abs(w.sum() - 1.0) < 1e-12


@pytest.mark.parametrize("d_p,U", [(2, 3), (4, 3), (3, 4), (8, 2), (16, 2), (4, 5)])
def test_full_product_equals_softmax_of_summed_logits(d_p, U):
    """The product of per-digit softmax probabilities over all M slots equals the softmax
    of the M summed logits (the factorisation the five views share).  Also pins the digit
    order: slot i's weight must belong to big-endian digits of i."""
    M = d_p ** U
    x = RNG.normal(0, 2.0, d_p * U)
    idx, _ = oracle.topk_bruteforce(x, d_p, U, M)
    w = oracle.weights(x, d_p, U, idx, renorm=0)
    ref = torch.softmax(torch.tensor(_summed_logits(x, d_p, U), dtype=torch.float64), 0).numpy()
    np.testing.assert_allclose(w, ref[idx], rtol=1e-12, atol=1e-15)
    assert abs(w.sum() - 1.0) < 1e-12


@pytest.mark.parametrize("d_p,U,K", [(4, 5, 8), (4, 5, 32), (8, 4, 16), (2, 6, 5), (16, 2, 7)])
def test_topk_is_top_of_product_probabilities(d_p, U, K):
    """Reading R3: ranking by the integer score is ranking by the product of digit
    probabilities.  On draws whose K-th and (K+1)-th fp64 products are clearly apart, the
    oracle's Top-K set equals the Top-K of the fp64 products computed by torch.softmax."""
    checked = 0
    for _ in range(60):
        x = RNG.normal(0, 1.5, d_p * U)
        s = _summed_logits(x, d_p, U)
        p = torch.softmax(torch.tensor(s), 0).numpy()
        order = np.argsort(-p, kind="stable")
        if K < p.size and p[order[K - 1]] - p[order[K]] < 1e-9 * p[order[K - 1]]:
            continue
        idx, _ = oracle.topk_bruteforce(x, d_p, U, K)
        assert idx.tolist() == order[:K].tolist()
        checked += 1
    assert checked > 40


def test_exact_ties_break_to_lower_index():
    """Reading R4 on a fully tied address: all slots score the same, so the Top-K is the K
    lowest slot indices in increasing order; after CAPE those indices are shifted."""
    x = np.zeros(4 * 5)
    idx, key = oracle.topk_bruteforce(x, 4, 5, 8)
    assert idx.tolist() == list(range(8)) and (key == 0).all()
    cfg = OracleConfig(d_p=4, U=5, K=8, d_v=1)
    ci, cw = oracle.decode_addresses(cfg, x.reshape(1, 1, 1, 20), pos0=np.array([1020]),
                                     cape_mask=np.array([1]))
    assert ci[0, 0, 0].tolist() == [(i + 1020) % 1024 for i in range(8)]
    np.testing.assert_allclose(cw[0, 0, 0], np.full(8, 1 / 8), rtol=1e-15)


def test_hand_worked_two_digit_example():
    """A 2-digit binary address (d_p = 2, U = 2, M = 4) worked by hand: logits (1, 0 | 0.5,
    0.25) give slot sums 1.5, 1.25, 0.5, 0.25, so the Top-3 is slots 0, 1, 2 and their
    weights are products of the two digit softmaxes."""
    x = np.array([1.0, 0.0, 0.5, 0.25])
    idx, _ = oracle.topk_bruteforce(x, 2, 2, 3)
    assert idx.tolist() == [0, 1, 2]
    e = math.e
    p0 = [e / (e + 1), 1 / (e + 1)]
    a, b = math.exp(0.5), math.exp(0.25)
    p1 = [a / (a + b), b / (a + b)]
    raw = [p0[0] * p1[0], p0[0] * p1[1], p0[1] * p1[0]]
    np.testing.assert_allclose(oracle.weights(x, 2, 2, idx, 0), raw, rtol=1e-14)
    np.testing.assert_allclose(oracle.weights(x, 2, 2, idx, 1), np.array(raw) / sum(raw), rtol=1e-14)


@pytest.mark.parametrize("d_p,U,K", [(4, 5, 8), (4, 5, 32), (4, 5, 1), (8, 4, 16), (2, 10, 64),
                                     (3, 4, 81), (5, 3, 7), (16, 4, 64), (4, 2, 16), (2, 1, 2)])
def test_tree_search_equals_bruteforce(d_p, U, K):
    """The page's exactness argument: keeping the K best partial addresses per level returns
    the exact Top-K.  Brute force (all M scored, full sort) must equal the level-by-level
    search bit for bit, including tie order, on smooth and heavily tied logits."""
    for trial in range(40):
        if trial % 3 == 0:
            x = RNG.integers(-2, 3, d_p * U) * 0.25          # many exact ties
        elif trial % 3 == 1:
            x = RNG.normal(0, 0.1, d_p * U).astype(np.float32)
        else:
            x = RNG.normal(0, 4.0, d_p * U)
        a = oracle.topk_bruteforce(x, d_p, U, K)
        b = oracle.topk_tree(x, d_p, U, K)
        assert a[0].tolist() == b[0].tolist()
        assert a[1].tolist() == b[1].tolist()


def test_single_digit_reduces_to_stable_sorted_softmax():
    """U = 1 is one softmax over d_p values: the Top-K is a stable descending sort of the
    logits and the raw weights are torch.softmax entries."""
    for trial in range(30):
        x = RNG.integers(-3, 4, 16) * 0.5 if trial % 2 else RNG.normal(size=16)
        idx, _ = oracle.topk_bruteforce(x, 16, 1, 6)
        assert idx.tolist() == np.argsort(-x, kind="stable")[:6].tolist()
        ref = torch.softmax(torch.tensor(x), 0).numpy()[idx]
        np.testing.assert_allclose(oracle.weights(x, 16, 1, idx, 0), ref, rtol=1e-13)


def test_regroupable_digits():
    """Regroupable Address view: merging two adjacent digits into one coarser digit leaves
    every slot weight unchanged.  decode(U=4, d_p=4, x) == decode(U=2, d_p=16, x') with
    x'[a*4 + b] = x_{2g}[a] + x_{2g+1}[b]; logits on a 2^-8 grid keep the sums exact."""
    for trial in range(30):
        x = np.round(RNG.normal(0, 2.0, 16) * 256) / 256
        xs = x.reshape(4, 4)
        merged = np.concatenate([(xs[2 * g][:, None] + xs[2 * g + 1][None, :]).reshape(-1)
                                 for g in range(2)])
        for K in (1, 8, 37, 256):
            a = oracle.topk_bruteforce(x, 4, 4, K)
            b = oracle.topk_bruteforce(merged, 16, 2, K)
            assert a[0].tolist() == b[0].tolist() and a[1].tolist() == b[1].tolist()
            for rn in (0, 1):
                np.testing.assert_allclose(oracle.weights(x, 4, 4, a[0], rn),
                                           oracle.weights(merged, 16, 2, b[0], rn), rtol=1e-12)


def test_digit_score_grid():
    """Reading R3's integer score: x * 2^32 rounded half-to-even, clamped to +-4095, NaN
    lowest.  bf16-representable values land on the grid exactly."""
    assert oracle.digit_score(1.0) == 2 ** 32
    assert oracle.digit_score(-0.5) == -(2 ** 31)
    assert oracle.digit_score(2.0 ** -33) == 0          # half of one step -> even (0)
    assert oracle.digit_score(3 * 2.0 ** -33) == 2      # 1.5 steps -> 2
    assert oracle.digit_score(1e9) == 4095 * 2 ** 32
    assert oracle.digit_score(float("-inf")) == -4095 * 2 ** 32
    assert oracle.digit_score(float("nan")) == -4095 * 2 ** 32
    vals = torch.randn(1000).to(torch.bfloat16).double().numpy()
    for v in vals[np.abs(vals) >= 2.0 ** -25]:
        assert oracle.digit_score(v) == int(v * 2 ** 32)


# ------------------------------------------------------------------ CAPE

def test_cape_is_cyclic_permutation():
    """CAPE paragraphs: the shift wraps around the slot array and only permutes indices."""
    M = 64
    for pos in (0, 1, 63, 64, 1000, -5):
        shifted = [oracle.cape(i, pos, M) for i in range(M)]
        assert sorted(shifted) == list(range(M))
        assert shifted[0] == pos % M
    assert oracle.cape(M - 1, 1, M) == 0


def _scan_inputs(B, T, H, cfg, seed, std=1.5):
    r = np.random.default_rng(seed)
    k = r.normal(0, std, (B, T, H, cfg.L))
    q = r.normal(0, std, (B, T, H, cfg.L))
    v = r.normal(size=(B, T, H, cfg.d_v))
    g = 1 / (1 + np.exp(-r.normal(size=(B, T, H))))
    z = 1 / (1 + np.exp(-r.normal(size=(B, T, H, cfg.d_v))))
    return k, q, v, g, z


def test_cape_relative_position_equivariance():
    """CAPE paragraphs: overlap between a read at t and a write at s depends on content and
    t - s only.  Starting every sequence at position P instead of 0 (zero initial state,
    CAPE on all heads) must give bit-identical outputs and a state rolled by P slots."""
    cfg = OracleConfig(d_p=2, U=5, K=4, d_v=8)
    k, q, v, g, z = _scan_inputs(2, 40, 2, cfg, 7)
    mask = np.ones(2, np.uint8)
    y0, S0, m0 = oracle.scan_forward(cfg, k, q, v, g, z, cape_mask=mask, pos0=np.array([0, 0]))
    P = np.array([5, 1000])
    y1, S1, m1 = oracle.scan_forward(cfg, k, q, v, g, z, cape_mask=mask, pos0=P)
    assert np.array_equal(y0, y1)
    for b in range(2):
        assert np.array_equal(np.roll(S0[b], P[b] % cfg.M, axis=1), S1[b])
        assert np.array_equal(np.roll(m0[b], P[b] % cfg.M, axis=1), m1[b])


def test_cape_mask_leaves_content_heads_unshifted():
    """CAPE applies to some heads only; content-only heads do not depend on position."""
    cfg = OracleConfig(d_p=4, U=3, K=4, d_v=8)
    k, q, v, g, z = _scan_inputs(1, 30, 3, cfg, 8)
    mask = np.array([1, 0, 1], np.uint8)
    ya, Sa, _ = oracle.scan_forward(cfg, k, q, v, g, z, cape_mask=mask, pos0=np.array([0]))
    yb, Sb, _ = oracle.scan_forward(cfg, k, q, v, g, z, cape_mask=mask, pos0=np.array([17]))
    assert np.array_equal(ya[:, :, 1], yb[:, :, 1]) and np.array_equal(Sa[:, 1], Sb[:, 1])
    assert np.array_equal(np.roll(Sa[:, 0], 17, axis=1), Sb[:, 0])
    y_off, S_off, _ = oracle.scan_forward(cfg, k, q, v, g, z, cape_mask=None)
    assert np.array_equal(y_off[:, :, 1], ya[:, :, 1])


# ------------------------------------------------------------------ Gated Sparse Update

@pytest.mark.parametrize("w,g,expect", [
    (0.0, 0.7, 1.0), (0.0, 1.0, 1.0), (0.4, 0.0, 1.0), (0.3, 1.0, 0.0), (1.0, 0.2, 0.0),
    (0.5, 0.5, 0.5), (0.25, 2 / 3, 0.5625), (0.5, 0.2, 0.5 ** 0.25), (0.9, 0.9, 0.1 ** 9),
    (0.5, float("nan"), 1.0), (0.5, 1.5, 0.0), (0.5, -0.3, 1.0)])
def test_alpha_edge_table(w, g, expect):
    """Gated Sparse Update step 1 and its limits: no write keeps everything (w = 0 -> 1),
    gamma -> -inf keeps everything (g = 0), gamma -> +inf keeps nothing (g = 1); in between
    (1 - w) ** e^gamma with e^gamma = g / (1 - g)."""
    assert oracle.alpha(w, g) == pytest.approx(expect, rel=1e-12, abs=1e-300)


def test_alpha_monotone_in_write_and_gate():
    """Step 1: a stronger write or a larger gamma keeps less of the old mass."""
    ws = np.linspace(0.01, 0.99, 25)
    gs = np.linspace(0.01, 0.99, 25)
    A = np.array([[oracle.alpha(w, g) for g in gs] for w in ws])
    assert (np.diff(A, axis=0) < 0).all() and (np.diff(A, axis=1) < 0).all()


def test_unselected_slots_unchanged():
    """Gated Sparse Update: slots with no write keep content and mass bit for bit."""
    cfg = OracleConfig(d_p=4, U=4, K=8, d_v=8)
    B, T, H = 2, 50, 2
    k, q, v, g, z = _scan_inputs(B, T, H, cfg, 9)
    r = np.random.default_rng(10)
    S_in = r.normal(size=(B, H, cfg.M, cfg.d_v))
    m_in = r.uniform(0.5, 2, (B, H, cfg.M))
    mask = np.array([1, 0], np.uint8)
    pos0 = np.array([3, 900], np.int32)
    _, S, m = oracle.scan_forward(cfg, k, q, v, g, z, cape_mask=mask, pos0=pos0, S_in=S_in, m_in=m_in)
    wi, _ = oracle.decode_addresses(cfg, k, pos0=pos0, cape_mask=mask)
    for b in range(B):
        for h in range(H):
            written = np.zeros(cfg.M, bool)
            written[wi[b, :, h].reshape(-1)] = True
            assert written.sum() < cfg.M
            assert np.array_equal(S[b, h, ~written], S_in[b, h, ~written])
            assert np.array_equal(m[b, h, ~written], m_in[b, h, ~written])
            assert not np.array_equal(S[b, h, written], S_in[b, h, written])


def _write_history(cfg, k, pos0=None, cape_mask=None):
    wi, ww = oracle.decode_addresses(cfg, k, pos0=pos0, cape_mask=cape_mask)
    return wi, ww


def test_gate_zero_is_running_weighted_average():
    """gamma -> -inf (g = 0): GSU averages all past writes.  From a zero state the slot is
    sum_s w_s v_s / (sum_s w_s + eps) and its mass is sum_s w_s."""
    cfg = OracleConfig(d_p=4, U=3, K=4, d_v=6)
    B, T, H = 1, 80, 1
    k, q, v, g, z = _scan_inputs(B, T, H, cfg, 11)
    g[:] = 0.0
    _, S, m = oracle.scan_forward(cfg, k, q, v, g, z)
    wi, ww = _write_history(cfg, k)
    num = np.zeros((cfg.M, cfg.d_v))
    den = np.zeros(cfg.M)
    for t in range(T):
        for j in range(cfg.K):
            num[wi[0, t, 0, j]] += ww[0, t, 0, j] * v[0, t, 0]
            den[wi[0, t, 0, j]] += ww[0, t, 0, j]
    np.testing.assert_allclose(m[0, 0], den, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(S[0, 0], num / (den + cfg.eps_gsu)[:, None], rtol=1e-10, atol=1e-13)


def test_gate_one_overwrites_with_newest():
    """gamma -> +inf (g = 1): the mass is the newest write weight and the slot content is
    the newest value up to the eps share eps / (w + eps) of the previous content."""
    cfg = OracleConfig(d_p=4, U=3, K=4, d_v=6)
    B, T, H = 1, 60, 1
    k, q, v, g, z = _scan_inputs(B, T, H, cfg, 12)
    g[:] = 1.0
    r = np.random.default_rng(13)
    S_in = r.normal(size=(B, H, cfg.M, cfg.d_v))
    _, S, m = oracle.scan_forward(cfg, k, q, v, g, z, S_in=S_in)
    wi, ww = _write_history(cfg, k)
    last_w = {}
    last_v = {}
    for t in range(T):
        for j in range(cfg.K):
            last_w[wi[0, t, 0, j]] = ww[0, t, 0, j]
            last_v[wi[0, t, 0, j]] = v[0, t, 0]
    bound = np.abs(S_in).max() + np.abs(v).max()
    for i, w in last_w.items():
        assert m[0, 0, i] == pytest.approx(w, rel=1e-15)
        assert np.abs(S[0, 0, i] - last_v[i]).max() <= cfg.eps_gsu / (w + cfg.eps_gsu) * bound * 1.0001


def test_slots_are_bounded_averages():
    """Slots stay bounded averages: every channel of a slot lies between the smallest and
    largest of its initial value and the values written into it."""
    cfg = OracleConfig(d_p=4, U=3, K=6, d_v=5)
    B, T, H = 1, 120, 2
    k, q, v, g, z = _scan_inputs(B, T, H, cfg, 14)
    r = np.random.default_rng(15)
    S_in = r.uniform(-1, 1, (B, H, cfg.M, cfg.d_v))
    _, S, _ = oracle.scan_forward(cfg, k, q, v, g, z, S_in=S_in)
    wi, _ = _write_history(cfg, k)
    for h in range(H):
        lo = S_in[0, h].copy()
        hi = S_in[0, h].copy()
        for t in range(T):
            for i in wi[0, t, h]:
                lo[i] = np.minimum(lo[i], v[0, t, h])
                hi[i] = np.maximum(hi[i], v[0, t, h])
        assert (S[0, h] >= lo - 1e-12).all() and (S[0, h] <= hi + 1e-12).all()


def test_mass_recurrence_worked_example():
    """One slot written twice with known weights: d_p = 2, U = 1, K = 1, raw weights.
    Logits (ln 3, 0) select slot 0 with w = 3/4; g = 1/2 gives e^gamma = 1 and
    alpha = 1/4.  Mass 3/4 then 1/4 * 3/4 + 3/4 = 15/16; content follows step 4."""
    cfg = OracleConfig(d_p=2, U=1, K=1, d_v=2, renorm=0)
    k = np.array([math.log(3), 0.0] * 2).reshape(1, 2, 1, 2)
    v = np.array([[1.0, -2.0], [3.0, 5.0]]).reshape(1, 2, 1, 2)
    g = np.full((1, 2, 1), 0.5)
    z = np.ones((1, 2, 1, 2))
    y, S, m = oracle.scan_forward(cfg, k, k, v, g, z)
    eps = cfg.eps_gsu
    lam0 = 0.75 / (0.75 + eps)
    s0 = lam0 * v[0, 0, 0]
    lam1 = 0.75 / (15 / 16 + eps)
    s1 = s0 + lam1 * (v[0, 1, 0] - s0)
    assert m[0, 0, 0] == pytest.approx(15 / 16, rel=1e-15) and m[0, 0, 1] == 0
    np.testing.assert_allclose(S[0, 0, 0], s1, rtol=1e-14)
    # read after write: the token reads its own slot with raw weight 3/4
    o1 = 0.75 * s1
    np.testing.assert_allclose(y[0, 1, 0], o1 / np.sqrt((o1 ** 2).mean() + cfg.eps_norm), rtol=1e-13)


# ------------------------------------------------------------------ read, norm, gate

def test_read_sees_this_tokens_write():
    """Reading R10: a token whose query addresses the slots its key writes, with g = 1
    (overwrite) and a negligible eps, reads back its own value: y = v / rms(v) * z."""
    cfg = OracleConfig(d_p=4, U=3, K=4, d_v=16, eps_gsu=1e-300, eps_norm=1e-300)
    k, q, v, g, z = _scan_inputs(1, 20, 1, cfg, 16)
    g[:] = 1.0
    S_in = np.random.default_rng(17).normal(size=(1, 1, cfg.M, cfg.d_v)) * 10
    y, _, _ = oracle.scan_forward(cfg, k, k, v, g, z, S_in=S_in)
    vv = v[0, :, 0]
    ref = vv / np.sqrt((vv ** 2).mean(-1, keepdims=True)) * z[0, :, 0]
    np.testing.assert_allclose(y[0, :, 0], ref, rtol=1e-9, atol=1e-12)


def test_rmsnorm_and_gate():
    """Output RMSNorm and gate: y / z has root-mean-square sqrt(ms / (ms + eps)) ~ 1, is
    invariant to scaling the values (the state is linear in v from a zero start), and a
    norm weight multiplies each channel."""
    cfg = OracleConfig(d_p=4, U=3, K=4, d_v=16)
    k, q, v, g, z = _scan_inputs(1, 40, 2, cfg, 18)
    y, _, _ = oracle.scan_forward(cfg, k, q, v, g, z)
    rms = np.sqrt(((y / z) ** 2).mean(-1))
    live = rms > 0
    assert live.mean() > 0.8
    np.testing.assert_allclose(rms[live], 1.0, atol=1e-4)
    y1000, _, _ = oracle.scan_forward(cfg, k, q, v * 1000, g, z)
    y2000, _, _ = oracle.scan_forward(cfg, k, q, v * 2000, g, z)
    np.testing.assert_allclose(y1000, y2000, rtol=1e-9, atol=1e-12)
    nw = np.linspace(0.5, 2.0, cfg.d_v)
    yw, _, _ = oracle.scan_forward(cfg, k, q, v, g, z, norm_w=nw)
    np.testing.assert_allclose(yw, y * nw, rtol=1e-13, atol=1e-15)


# ------------------------------------------------------------------ state carry

def test_chunked_scan_and_decode_chain_equal_full_scan():
    """The recurrent state is the checkpoint: scan(T) == scan(T1) then scan(T - T1) with the
    state and start position carried, and == T single decode steps."""
    cfg = OracleConfig(d_p=4, U=3, K=4, d_v=8)
    B, T, H = 2, 30, 2
    k, q, v, g, z = _scan_inputs(B, T, H, cfg, 19)
    mask = np.array([1, 0], np.uint8)
    pos0 = np.array([0, 77], np.int32)
    y, S, m = oracle.scan_forward(cfg, k, q, v, g, z, cape_mask=mask, pos0=pos0)
    T1 = 13
    ya, Sa, ma = oracle.scan_forward(cfg, k[:, :T1], q[:, :T1], v[:, :T1], g[:, :T1], z[:, :T1],
                                     cape_mask=mask, pos0=pos0)
    yb, Sb, mb = oracle.scan_forward(cfg, k[:, T1:], q[:, T1:], v[:, T1:], g[:, T1:], z[:, T1:],
                                     cape_mask=mask, pos0=pos0 + T1, S_in=Sa, m_in=ma)
    assert np.array_equal(np.concatenate([ya, yb], 1), y)
    assert np.array_equal(Sb, S) and np.array_equal(mb, m)
    Sd = np.zeros_like(S)
    md = np.zeros_like(m)
    for t in range(T):
        yd = oracle.decode_step(cfg, k[:, t], q[:, t], v[:, t], g[:, t], z[:, t], Sd, md,
                                pos=pos0 + t, cape_mask=mask)
        assert np.array_equal(yd, y[:, t])
    assert np.array_equal(Sd, S) and np.array_equal(md, m)


def test_decode_step_unit_range_touches_only_its_units():
    cfg = OracleConfig(d_p=4, U=3, K=4, d_v=8)
    k, q, v, g, z = _scan_inputs(3, 1, 2, cfg, 20)
    S = np.random.default_rng(21).normal(size=(3, 2, cfg.M, cfg.d_v))
    m = np.ones((3, 2, cfg.M))
    S0, m0 = S.copy(), m.copy()
    y = oracle.decode_step(cfg, k[:, 0], q[:, 0], v[:, 0], g[:, 0], z[:, 0], S, m, units=(2, 4))
    flat_S, flat_S0 = S.reshape(6, -1), S0.reshape(6, -1)
    for u in range(6):
        assert np.array_equal(flat_S[u], flat_S0[u]) == (u not in (2, 3))
    assert (y.reshape(6, -1)[[0, 1, 4, 5]] == 0).all()


# ------------------------------------------------------------------ state-access accounting

def test_state_access_accounting_matches_page(golden_dir):
    """GPU execution paragraph: per decode step a head touches 2*K*d_v state elements
    (K read rows + K write rows) out of M*d_v; with M = 1024 and d_v = 128 this
    reproduces the page's 0.4M of 26.2M (340M, Top-8), 0.8M of 52.4M and 1.6M (1.3B)."""
    M, d_v = 1024, 128
    for kind, f in _read_facts(golden_dir):
        if kind != "state_access":
            continue
        n_heads = round(float(f["total"]) * 1e6 / (M * d_v))
        assert abs(n_heads * M * d_v / 1e6 - float(f["total"])) < 0.05
        active = n_heads * 2 * int(f["K"]) * d_v
        assert round(active / 1e6, 1) == float(f["active"])
