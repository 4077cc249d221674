"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Indices must match bit for bit (including rank order); floating outputs and final state
within max-abs 1e-5 when every input is fp32 and 1e-3 with bf16 inputs (fp32 state).
Small cases are compared element by element; the full-size workloads run in the launch
configuration bench.py times and are compared on sampled tokens / heads, which the
oracle computes one at a time.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_slot_recurrent_b200 import ramnet
from sparse_slot_recurrent_b200.workloads import WORKLOADS, Workload, generate, generate_decode_state

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
TOL_BF16 = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    ramnet.load()
    yield
    ramnet.sync_status()


def _cfgs(w: Workload, **kw):
    c = dict(d_p=w.d_p, U=w.U, K=w.K, d_v=w.d_v)
    c.update(kw)
    return ramnet.Config(**c), oracle.OracleConfig(**c)


def _tol(dtype):
    return TOL_F32 if dtype == torch.float32 else TOL_BF16


def _cuda(inp):
    return {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items() if not k.startswith("_")}


def _maxabs(a, b):
    a = a.detach().cpu().double().numpy() if torch.is_tensor(a) else a
    b = b.detach().cpu().double().numpy() if torch.is_tensor(b) else b
    return float(np.abs(a - b).max()) if a.size else 0.0


# ------------------------------------------------------------------ address decoder

DECODE_CASES = [
    # d_p, U, K, dtype, logit mode
    (4, 5, 8, torch.float32, "normal"),
    (4, 5, 8, torch.bfloat16, "ties"),
    (4, 5, 32, torch.bfloat16, "mixed"),
    (8, 4, 16, torch.bfloat16, "normal"),
    (2, 8, 64, torch.float32, "ties"),
    (16, 4, 64, torch.bfloat16, "normal"),
    (3, 4, 17, torch.float32, "ties"),
    (5, 3, 7, torch.bfloat16, "normal"),
    (16, 2, 1, torch.float32, "normal"),
    (2, 1, 2, torch.float32, "ties"),
]


def _logits(B, T, H, L, mode, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    if mode == "ties":
        x = torch.randint(-2, 3, (B, T, H, L), generator=g).float() * 0.25
    elif mode == "mixed":
        x = torch.randn((B, T, H, L), generator=g)
        peaked = torch.rand((B, T, H, 1), generator=g) < 0.7
        x = x * torch.where(peaked, torch.tensor(4.0), torch.tensor(0.1))
    else:
        x = torch.randn((B, T, H, L), generator=g) * 1.5
    return x.to(dtype).contiguous()


@pytest.mark.parametrize("d_p,U,K,dtype,mode", DECODE_CASES)
def test_decode_addresses_matches_oracle(d_p, U, K, dtype, mode):
    B, T, H = 2, 37, 3
    cfg = ramnet.Config(d_p=d_p, U=U, K=K, d_v=16)
    ocfg = oracle.OracleConfig(d_p=d_p, U=U, K=K, d_v=16)
    x = _logits(B, T, H, d_p * U, mode, dtype, seed=d_p * 100 + K)
    pos0 = torch.tensor([0, 1234567], dtype=torch.int32)
    mask = torch.tensor([1, 0, 1], dtype=torch.uint8)
    for renorm in (1, 0):
        cfg_r = ramnet.Config(d_p=d_p, U=U, K=K, d_v=16, renorm=renorm)
        ocfg_r = oracle.OracleConfig(d_p=d_p, U=U, K=K, d_v=16, renorm=renorm)
        idx, w = ramnet.decode_addresses(cfg_r, x.cuda(), pos0=pos0.cuda(), cape_mask=mask.cuda())
        oi, ow = oracle.decode_addresses(ocfg_r, x, pos0=pos0, cape_mask=mask)
        assert np.array_equal(idx.cpu().numpy(), oi)
        assert _maxabs(w, ow) <= 2e-6
    del cfg, ocfg


def test_decode_addresses_strided_views():
    """Logits handed over as non-contiguous views (ramnet_strides): a [B,H,T,L] array read as
    [B,T,H,L], and a slice of wider rows starting at an odd element."""
    d_p, U, K = 4, 5, 16
    cfg = ramnet.Config(d_p=d_p, U=U, K=K, d_v=16)
    ocfg = oracle.OracleConfig(d_p=d_p, U=U, K=K, d_v=16)
    B, T, H, L = 2, 45, 3, d_p * U
    pos0 = torch.tensor([7, 100], dtype=torch.int32)
    mask = torch.tensor([1, 0, 1], dtype=torch.uint8)
    base = _logits(B, H, T, L, "ties", torch.bfloat16, seed=77).cuda()  # [B,H,T,L]
    wide = _logits(B, T, H, L + 9, "normal", torch.bfloat16, seed=78).cuda()
    for xd in (base.permute(0, 2, 1, 3), wide[..., 3:3 + L]):
        assert not xd.is_contiguous() and xd.stride(-1) == 1
        idx, w = ramnet.decode_addresses(cfg, xd, pos0=pos0.cuda(), cape_mask=mask.cuda())
        oi, ow = oracle.decode_addresses(ocfg, xd.cpu().contiguous(), pos0=pos0, cape_mask=mask)
        assert np.array_equal(idx.cpu().numpy(), oi)
        assert _maxabs(w, ow) <= 2e-6


@pytest.mark.parametrize("name", ["prefill_340m_top8", "prefill_340m_top32", "prefill_1p3b_top16"])
def test_decode_addresses_full_size_sampled(name):
    w = WORKLOADS[name]
    cfg, ocfg = _cfgs(w)
    inp = generate(w, seed=0)
    rng = np.random.default_rng(5)
    for key in ("k_logits", "q_logits"):
        x = inp[key]
        idx, wt = ramnet.decode_addresses(cfg, x.cuda(), pos0=inp["pos0"].cuda(), cape_mask=inp["cape_mask"].cuda())
        idx, wt = idx.cpu(), wt.cpu()
        bs = rng.integers(0, w.B, 1500)
        ts = rng.integers(0, w.T, 1500)
        hs = rng.integers(0, w.H, 1500)
        sub = x[bs, ts, hs].reshape(1500, 1, 1, -1)
        pos = (inp["pos0"][bs].numpy() + ts).astype(np.int32)
        for n in range(1500):
            oi, ow = oracle.decode_addresses(ocfg, sub[n:n + 1], pos0=pos[n:n + 1],
                                             cape_mask=inp["cape_mask"][hs[n]:hs[n] + 1])
            assert np.array_equal(idx[bs[n], ts[n], hs[n]].numpy(), oi[0, 0, 0]), (key, n)
            assert _maxabs(wt[bs[n], ts[n], hs[n]], ow[0, 0, 0]) <= 2e-6


# ------------------------------------------------------------------ prefill scan

def _oracle_scan(ocfg, inp, norm_w=None, S_in=None, m_in=None):
    return oracle.scan_forward(ocfg, inp["k_logits"], inp["q_logits"], inp["v"], inp["g"], inp["z"],
                               norm_w=norm_w, cape_mask=inp["cape_mask"], pos0=inp["pos0"], S_in=S_in, m_in=m_in)


def _gpu_scan(cfg, inp, norm_w=None, S_in=None, m_in=None, out_dtype=torch.float32):
    d = _cuda(inp)
    y, S, m = ramnet.scan_forward(cfg, d["k_logits"], d["q_logits"], d["v"], d["g"], d["z"],
                                  norm_w=None if norm_w is None else norm_w.cuda(), cape_mask=d["cape_mask"],
                                  pos0=d["pos0"], S_in=None if S_in is None else S_in.cuda(),
                                  m_in=None if m_in is None else m_in.cuda(), out_dtype=out_dtype)
    ramnet.sync_status()
    return y.cpu(), S.cpu(), m.cpu()


def test_scan_tiny_all_fp32():
    """The all-fp32 tiny workload, every output element and the final state."""
    w = WORKLOADS["tiny"]
    cfg, ocfg = _cfgs(w)
    inp = generate(w, seed=0)
    y, S, m = _gpu_scan(cfg, inp)
    oy, oS, om = _oracle_scan(ocfg, inp)
    assert _maxabs(y, oy) <= TOL_F32
    assert _maxabs(S, oS) <= TOL_F32
    assert _maxabs(m, om) <= TOL_F32


SCAN_CASES = [
    # d_p, U, K, d_v, B, T, H, dtype, cape, with_state, norm_w
    (4, 5, 8, 128, 2, 211, 3, torch.bfloat16, "mixed", True, True),
    (4, 5, 32, 128, 1, 150, 2, torch.bfloat16, "off", False, False),
    (4, 5, 16, 64, 1, 100, 2, torch.float32, "all", True, False),
    (8, 4, 16, 128, 1, 70, 1, torch.bfloat16, "all", False, False),
    (4, 4, 8, 32, 2, 90, 2, torch.float32, "mixed", True, True),
    (2, 8, 64, 16, 1, 80, 1, torch.float32, "off", False, False),
    (4, 5, 1, 128, 1, 64, 1, torch.float32, "all", True, False),
    (16, 2, 8, 256, 1, 60, 1, torch.bfloat16, "off", True, True),
    (3, 5, 7, 32, 1, 77, 2, torch.float32, "mixed", False, False),
    (4, 5, 8, 128, 1, 1, 1, torch.float32, "all", True, False),
]


def _small_inputs(d_p, U, K, d_v, B, T, H, dtype, cape, seed):
    w = Workload("case", B=B, H=H, T=T, d_p=d_p, U=U, K=K, d_v=d_v, in_dtype=dtype, cape=cape != "off",
                 logit_std=1.5)
    inp = generate(w, seed=seed)
    if cape == "mixed":
        inp["cape_mask"] = torch.tensor([(h + 1) % 2 for h in range(H)], dtype=torch.uint8)
    inp["pos0"] = torch.arange(B, dtype=torch.int32) * 1000 + 3
    return w, inp


@pytest.mark.parametrize("case", SCAN_CASES)
def test_scan_matches_oracle(case):
    d_p, U, K, d_v, B, T, H, dtype, cape, with_state, with_nw = case
    w, inp = _small_inputs(d_p, U, K, d_v, B, T, H, dtype, cape, seed=K + d_v)
    cfg, ocfg = _cfgs(w)
    g = torch.Generator().manual_seed(99)
    S_in = torch.randn((B, H, w.M, d_v), generator=g) if with_state else None
    m_in = torch.rand((B, H, w.M), generator=g) * 2 if with_state else None
    nw = torch.rand(d_v, generator=g) + 0.5 if with_nw else None
    y, S, m = _gpu_scan(cfg, inp, nw, S_in, m_in)
    oy, oS, om = _oracle_scan(ocfg, inp, nw, S_in, m_in)
    tol = _tol(dtype)
    assert _maxabs(y, oy) <= tol
    assert _maxabs(S, oS) <= tol
    assert _maxabs(m, om) <= tol


def test_scan_raw_product_softmax_weights():
    """renorm = 0 (weights are the raw truncated product softmax) through the whole scan."""
    w, inp = _small_inputs(4, 5, 8, 64, 1, 150, 2, torch.float32, "mixed", seed=31)
    cfg, ocfg = _cfgs(w, renorm=0)
    g = torch.Generator().manual_seed(32)
    S_in = torch.randn((1, 2, w.M, 64), generator=g)
    m_in = torch.rand((1, 2, w.M), generator=g)
    y, S, m = _gpu_scan(cfg, inp, None, S_in, m_in)
    oy, oS, om = _oracle_scan(ocfg, inp, None, S_in, m_in)
    assert _maxabs(y, oy) <= TOL_F32
    assert _maxabs(S, oS) <= TOL_F32
    assert _maxabs(m, om) <= TOL_F32


def test_scan_route_then_recur_matches_oracle_and_forward():
    """The two-launch form (route, then recurrence over the workspace) gives the oracle's
    results and, bit for bit, the single-call results; a second recurrence over the same
    workspace gives the same bits again (every sum on the path has a fixed order)."""
    w, inp = _small_inputs(4, 4, 16, 64, 2, 233, 2, torch.bfloat16, "normal", seed=21)
    cfg, ocfg = _cfgs(w)
    g = torch.Generator().manual_seed(22)
    S_in = torch.randn((2, 2, w.M, 64), generator=g)
    m_in = torch.rand((2, 2, w.M), generator=g) * 2
    y0, S0, m0 = _gpu_scan(cfg, inp, None, S_in, m_in)
    d = _cuda(inp)
    ws = torch.empty(ramnet.scan_workspace_bytes(cfg, 2, 233, 2), dtype=torch.uint8, device="cuda")
    y = torch.empty((2, 233, 2, 64), dtype=torch.float32, device="cuda")
    S = torch.empty((2, 2, w.M, 64), dtype=torch.float32, device="cuda")
    m = torch.empty((2, 2, w.M), dtype=torch.float32, device="cuda")
    ramnet.scan_route(cfg, d["k_logits"], d["q_logits"], d["g"], ws, cape_mask=d["cape_mask"], pos0=d["pos0"])
    ramnet.scan_recur(cfg, d["v"], d["z"], y, S, m, ws, S_in=S_in.cuda(), m_in=m_in.cuda())
    ramnet.sync_status()
    oy, oS, om = _oracle_scan(ocfg, inp, None, S_in, m_in)
    assert _maxabs(y, oy) <= TOL_BF16 and _maxabs(S, oS) <= TOL_BF16 and _maxabs(m, om) <= TOL_BF16
    assert torch.equal(S.cpu(), S0.cpu()) and torch.equal(m.cpu(), m0.cpu())
    assert torch.equal(y.cpu(), y0.cpu())
    y2, S2, m2 = torch.full_like(y, float("nan")), torch.full_like(S, float("nan")), torch.full_like(m, float("nan"))
    ramnet.scan_recur(cfg, d["v"], d["z"], y2, S2, m2, ws, S_in=S_in.cuda(), m_in=m_in.cuda())
    ramnet.sync_status()
    assert torch.equal(y2, y) and torch.equal(S2, S) and torch.equal(m2, m)


def test_scan_unselected_slots_bit_identical():
    """Rows and masses of slots no token writes come back exactly as they went in."""
    w, inp = _small_inputs(4, 5, 8, 128, 2, 96, 2, torch.bfloat16, "mixed", seed=3)
    cfg, _ = _cfgs(w)
    g = torch.Generator().manual_seed(4)
    S_in = torch.randn((2, 2, w.M, 128), generator=g)
    m_in = torch.rand((2, 2, w.M), generator=g)
    _, S, m = _gpu_scan(cfg, inp, None, S_in, m_in)
    idx, _ = ramnet.decode_addresses(cfg, inp["k_logits"].cuda(), pos0=inp["pos0"].cuda(),
                                     cape_mask=inp["cape_mask"].cuda())
    idx = idx.cpu()
    for b in range(2):
        for h in range(2):
            written = torch.zeros(w.M, dtype=torch.bool)
            written[idx[b, :, h].reshape(-1).long()] = True
            assert (~written).sum() > 100
            assert torch.equal(S[b, h][~written], S_in[b, h][~written])
            assert torch.equal(m[b, h][~written], m_in[b, h][~written])


def test_scan_bf16_output_is_rounded_fp32_output():
    """Every bf16 output element is the round-to-nearest-even of the fp32 output element of
    the same call (the path is deterministic), and the fp32 output is within tolerance of the
    oracle, so each bf16 element is within one bf16 rounding of the oracle's value."""
    w, inp = _small_inputs(4, 5, 8, 128, 1, 130, 2, torch.bfloat16, "off", seed=6)
    cfg, ocfg = _cfgs(w)
    yb, Sb, mb = _gpu_scan(cfg, inp, out_dtype=torch.bfloat16)
    yf, Sf, mf = _gpu_scan(cfg, inp, out_dtype=torch.float32)
    assert torch.equal(yb, yf.to(torch.bfloat16))
    assert torch.equal(Sb, Sf) and torch.equal(mb, mf)
    oy, _, _ = _oracle_scan(ocfg, inp)
    assert _maxabs(yf, oy) <= TOL_BF16


def test_scan_state_carry_matches_single_call():
    """scan(T) == scan(T1) then scan(T - T1) with the state and start position carried."""
    w, inp = _small_inputs(4, 5, 8, 128, 1, 200, 2, torch.float32, "all", seed=7)
    cfg, _ = _cfgs(w)
    y, S, m = _gpu_scan(cfg, inp)
    T1 = 77
    a = {k: (v[:, :T1] if torch.is_tensor(v) and v.dim() >= 3 else v) for k, v in inp.items()}
    b = {k: (v[:, T1:].contiguous() if torch.is_tensor(v) and v.dim() >= 3 else v) for k, v in inp.items()}
    a = {k: (v.contiguous() if torch.is_tensor(v) else v) for k, v in a.items()}
    b["pos0"] = inp["pos0"] + T1
    ya, Sa, ma = _gpu_scan(cfg, a)
    yb, Sb, mb = _gpu_scan(cfg, b, S_in=Sa, m_in=ma)
    assert _maxabs(torch.cat([ya, yb], 1), y) <= TOL_F32
    assert _maxabs(Sb, S) <= TOL_F32 and _maxabs(mb, m) <= TOL_F32


@pytest.mark.parametrize("name", ["prefill_340m_top8", "prefill_340m_top32", "prefill_1p3b_top16"])
def test_scan_full_size_sampled_heads(name):
    """Full workload through the bench's launch configuration; two (b,h) heads compared
    with the oracle over the whole sequence; every head's never-written rows stay zero."""
    w = WORKLOADS[name]
    cfg, ocfg = _cfgs(w)
    inp = generate(w, seed=0)
    y, S, m = _gpu_scan(cfg, inp)
    tol = _tol(w.in_dtype)
    for (b, h) in [(0, 0), (w.B - 1, w.H - 1)]:
        sub = {k: inp[k][b:b + 1, :, h:h + 1].contiguous() for k in ("k_logits", "q_logits", "v", "z")}
        sub["g"] = inp["g"][b:b + 1, :, h:h + 1].contiguous()
        sub["cape_mask"] = inp["cape_mask"][h:h + 1]
        sub["pos0"] = inp["pos0"][b:b + 1]
        oy, oS, om = _oracle_scan(ocfg, sub)
        assert _maxabs(y[b:b + 1, :, h:h + 1], oy) <= tol
        assert _maxabs(S[b:b + 1, h:h + 1], oS) <= tol
        assert _maxabs(m[b:b + 1, h:h + 1], om) <= tol
    idx, _ = ramnet.decode_addresses(cfg, inp["k_logits"].cuda(), pos0=inp["pos0"].cuda(),
                                     cape_mask=inp["cape_mask"].cuda())
    written = torch.zeros((w.B, w.H, w.M), dtype=torch.bool, device="cuda")
    bi = torch.arange(w.B, device="cuda").view(w.B, 1, 1, 1).expand_as(idx)
    hi = torch.arange(w.H, device="cuda").view(1, 1, w.H, 1).expand_as(idx)
    written[bi.reshape(-1), hi.reshape(-1), idx.reshape(-1).long()] = True
    written = written.cpu()
    assert (S[~written] == 0).all() and (m[~written] == 0).all()


def _parse_route_workspace(cfg, dtype, ws, B, T, H):
    """Split the workspace written by ramnet_scan_route into per-head event arrays (see
    ramnet_scan_layout) and check its structure: per chunk the ranks' ranges tile the chunk's
    events, every event sits in the range of the scan warp that owns its slot, and each
    owner's events are in (token, stream) order."""
    lay = ramnet.scan_layout(cfg, dtype)
    C, ncta, nw, hw, K = lay.chunk, lay.ncta, lay.scan_warps, lay.hdr_words, cfg.K
    nch = -(-T // C)
    raw = ws.cpu().numpy()
    ev_bytes = B * H * nch * 2 * C * K * 16
    ev = raw[:ev_bytes].view(np.uint32).reshape(B * H, nch, 2 * C * K, 4)
    off = (ev_bytes + 255) // 256 * 256
    hdr = raw[off:off + B * H * nch * ncta * hw * 4].view(np.uint32).reshape(B * H, nch, ncta, hw)
    heads = {}
    for bh in range(B * H):
        rows = []
        nloc = np.zeros((nch * C, ncta), np.int64)
        for c in range(nch):
            nt = min(C, T - c * C)
            pos = 0
            for r in range(ncta):
                hd = hdr[bh, c, r]
                start, n = int(hd[0]), int(hd[1])
                assert start == pos and int(hd[2]) == nt and int(hd[3]) == 0
                pos += n
                woff = hd[4:4 + nw + 1].astype(np.int64)
                assert woff[0] == 0 and woff[-1] == n and np.all(np.diff(woff) >= 0)
                nloc[c * C:c * C + nt, r] = hd[4 + nw + 1:].view(np.uint8)[:nt]
                for wi in range(nw):
                    e = ev[bh, c, start + woff[wi]:start + woff[wi + 1]]
                    x = e[:, 0].astype(np.int64)
                    s, tl, q, st = x & 0xFFFF, (x >> 16) & 0xFF, (x >> 24) & 0x3F, x >> 31
                    slot = e[:, 3].astype(np.int64)
                    assert np.all(slot % ncta == r) and np.all(slot // ncta == s) and np.all(s % nw == wi)
                    assert np.all(tl < nt)
                    key = tl * 2 + st
                    assert np.all(np.diff(key) >= 0), "owner list out of (token, stream) order"
                    wt = e[:, 1].view(np.float32)
                    al = e[:, 2].view(np.float32)
                    ints = np.stack([c * C + tl, st, slot, q, np.full_like(tl, r)], 1).astype(np.int64)
                    rows.append((ints, wt.astype(np.float64), al.astype(np.float64)))
            assert pos == 2 * nt * K
        ints = np.concatenate([r[0] for r in rows])
        heads[bh] = (ints, np.concatenate([r[1] for r in rows]), np.concatenate([r[2] for r in rows]), nloc)
    return heads, ncta


def _check_route_head(ocfg, heads, ncta, bh, k_logits, q_logits, g, pos, cape_on, K):
    """One head's events against the oracle: write and read slot sets bit for bit, the
    per-rank read order (q) equal to the oracle's rank order, weights, retentions, and the
    per-rank read counts."""
    ints, wt, al, nloc = heads[bh]
    T = k_logits.shape[0]
    mask = np.array([1 if cape_on else 0], np.uint8)
    oi_k, ow_k = oracle.decode_addresses(ocfg, k_logits.reshape(1, T, 1, -1), pos0=np.array([pos], np.int32),
                                         cape_mask=mask)
    oi_q, ow_q = oracle.decode_addresses(ocfg, q_logits.reshape(1, T, 1, -1), pos0=np.array([pos], np.int32),
                                         cape_mask=mask)
    oi_k, ow_k, oi_q, ow_q = oi_k[0, :, 0], ow_k[0, :, 0], oi_q[0, :, 0], ow_q[0, :, 0]
    tok, st, slot, q, rk = ints.T
    # writes: per token the same slots (sorted), with the same weights
    wsel = st == 0
    o = np.lexsort((slot[wsel], tok[wsel]))
    osort = np.argsort(oi_k, axis=1, kind="stable")
    assert np.array_equal(slot[wsel][o], np.take_along_axis(oi_k, osort, 1).reshape(-1))
    exp_w = np.take_along_axis(ow_k, osort, 1).reshape(-1)
    assert np.abs(wt[wsel][o] - exp_w).max() <= 2e-6
    # retention of GSU step 1 from the same (fp32) weight and the token's gate
    gw = np.repeat(g.astype(np.float64), K)
    a_gpu, w_gpu = al[wsel][o], wt[wsel][o]
    for i in range(0, exp_w.size, max(1, exp_w.size // 3000)):
        assert abs(a_gpu[i] - oracle.alpha(w_gpu[i], gw[i])) <= 4e-6
    # reads: per token and rank, in q order, the oracle's reads of that rank in rank (j) order
    rsel = st == 1
    o = np.lexsort((q[rsel], rk[rsel], tok[rsel]))
    ork = oi_q % ncta
    osort = np.argsort(ork, axis=1, kind="stable")
    assert np.array_equal(slot[rsel][o], np.take_along_axis(oi_q, osort, 1).reshape(-1))
    assert np.abs(wt[rsel][o] - np.take_along_axis(ow_q, osort, 1).reshape(-1)).max() <= 2e-6
    assert np.all(al[rsel] == 0.0)
    cnt = np.stack([(ork == r).sum(1) for r in range(ncta)], 1)
    assert np.array_equal(nloc[:T], cnt)


ROUTE_CASES = [
    # d_p, U, K, d_v, B, T, H, dtype, logit mode, cape
    (4, 5, 8, 128, 1, 200, 2, torch.bfloat16, "normal", "mixed"),
    (4, 5, 8, 128, 1, 97, 1, torch.bfloat16, "ties", "all"),
    (4, 5, 16, 128, 1, 150, 2, torch.bfloat16, "ties", "off"),
    (4, 5, 32, 128, 1, 70, 1, torch.bfloat16, "mixed", "all"),
    (8, 4, 16, 128, 1, 40, 1, torch.bfloat16, "normal", "all"),
    (3, 4, 17, 32, 1, 60, 2, torch.float32, "ties", "mixed"),
    (2, 8, 64, 16, 1, 33, 1, torch.float32, "normal", "off"),
]


@pytest.mark.parametrize("case", ROUTE_CASES)
def test_route_events_match_oracle(case):
    """ramnet_scan_route's workspace, decoded: the hot path's Top-K (the register search for
    K <= 32), weights, CAPE and retentions bit-exact / within 2e-6 of the oracle, and the
    events bucketed by owning scan warp in causal order."""
    d_p, U, K, d_v, B, T, H, dtype, mode, cape = case
    cfg = ramnet.Config(d_p=d_p, U=U, K=K, d_v=d_v)
    ocfg = oracle.OracleConfig(d_p=d_p, U=U, K=K, d_v=d_v)
    kx = _logits(B, T, H, d_p * U, mode, dtype, seed=K * 7 + d_p)
    qx = _logits(B, T, H, d_p * U, mode, dtype, seed=K * 7 + d_p + 1)
    gg = torch.sigmoid(torch.randn((B, T, H), generator=torch.Generator().manual_seed(K))).to(dtype)
    mask = torch.tensor([1 if (cape == "all" or (cape == "mixed" and h % 2 == 0)) else 0 for h in range(H)],
                        dtype=torch.uint8)
    pos0 = torch.arange(B, dtype=torch.int32) * 977 + 5
    ws = torch.empty(ramnet.scan_workspace_bytes(cfg, B, T, H), dtype=torch.uint8, device="cuda")
    ramnet.scan_route(cfg, kx.cuda(), qx.cuda(), gg.cuda(), ws, cape_mask=mask.cuda(), pos0=pos0.cuda())
    ramnet.sync_status()
    heads, ncta = _parse_route_workspace(cfg, dtype, ws, B, T, H)
    for b in range(B):
        for h in range(H):
            _check_route_head(ocfg, heads, ncta, b * H + h, kx[b, :, h].double().numpy(), qx[b, :, h].double().numpy(),
                              gg[b, :, h].double().numpy(), int(pos0[b]), bool(mask[h]), K)


@pytest.mark.parametrize("name", ["prefill_340m_top8", "prefill_1p3b_top16", "prefill_340m_top32"])
def test_route_events_full_size_sampled_heads(name):
    """The full workload through ramnet_scan_route in the bench's launch configuration;
    two heads' events decoded and compared with the oracle over the whole sequence."""
    w = WORKLOADS[name]
    cfg, ocfg = _cfgs(w)
    inp = generate(w, seed=0)
    d = _cuda(inp)
    ws = torch.empty(ramnet.scan_workspace_bytes(cfg, w.B, w.T, w.H), dtype=torch.uint8, device="cuda")
    ramnet.scan_route(cfg, d["k_logits"], d["q_logits"], d["g"], ws, cape_mask=d["cape_mask"], pos0=d["pos0"])
    ramnet.sync_status()
    lay = ramnet.scan_layout(cfg, w.in_dtype)
    # parse only the sampled heads' part of the workspace
    nch = -(-w.T // lay.chunk)
    per_head_ev = nch * 2 * lay.chunk * w.K * 16
    ev_bytes = w.B * w.H * per_head_ev
    hdr_off = (ev_bytes + 255) // 256 * 256
    per_head_hdr = nch * lay.ncta * lay.hdr_words * 4
    for (b, h) in [(0, 1), (w.B - 1, w.H - 1)]:
        bh = b * w.H + h
        sub = torch.cat([ws[bh * per_head_ev:(bh + 1) * per_head_ev],
                         torch.zeros((-per_head_ev) % 256, dtype=torch.uint8, device="cuda"),
                         ws[hdr_off + bh * per_head_hdr:hdr_off + (bh + 1) * per_head_hdr]])
        heads, ncta = _parse_route_workspace(cfg, w.in_dtype, sub, 1, w.T, 1)
        _check_route_head(ocfg, heads, ncta, 0, inp["k_logits"][b, :, h].double().numpy(),
                          inp["q_logits"][b, :, h].double().numpy(), inp["g"][b, :, h].double().numpy(),
                          int(inp["pos0"][b]), bool(inp["cape_mask"][h]), w.K)


def test_decode_addresses_extreme_logits():
    """NaN, +-inf and |x| > 4095 logits: indices bit-exact with the oracle (NaN ranks lowest,
    values clamp at +-4095); weights compared where every logit of the token is within the
    clamp range (outside it the clamp enters the GPU weights by definition)."""
    for (d_p, U, K, dtype) in [(4, 5, 8, torch.float32), (4, 5, 16, torch.bfloat16), (8, 4, 16, torch.float32),
                               (4, 5, 32, torch.float32)]:
        B, T, H, L = 1, 300, 2, d_p * U
        g = torch.Generator().manual_seed(K + d_p)
        x = torch.randn((B, T, H, L), generator=g) * 2
        # about half of the tokens get extreme values in some of their logits
        pick = torch.rand((B, T, H, L), generator=g) + (torch.rand((B, T, H, 1), generator=g) < 0.5).float()
        x = torch.where(pick < 0.05, torch.tensor(float("nan")), x)
        x = torch.where((pick >= 0.05) & (pick < 0.08), torch.tensor(float("inf")), x)
        x = torch.where((pick >= 0.08) & (pick < 0.11), torch.tensor(float("-inf")), x)
        x = torch.where((pick >= 0.11) & (pick < 0.14), torch.tensor(1e6), x)
        x = torch.where((pick >= 0.14) & (pick < 0.17), torch.tensor(-5000.0), x)
        x = x.to(dtype)
        cfg = ramnet.Config(d_p=d_p, U=U, K=K, d_v=16)
        ocfg = oracle.OracleConfig(d_p=d_p, U=U, K=K, d_v=16)
        idx, w = ramnet.decode_addresses(cfg, x.cuda())
        oi, ow = oracle.decode_addresses(ocfg, x)
        assert np.array_equal(idx.cpu().numpy(), oi)
        tame = (x.double().abs() <= 4095).all(-1).numpy()
        assert tame.sum() > 100 and (~tame).sum() > 100
        assert np.abs(w.cpu().numpy()[tame] - ow[tame]).max() <= 2e-6


def test_scan_write_gate_edges():
    """Write gates exactly 0 (alpha = 1: running mean), exactly 1 (alpha = 0: overwrite) and
    a mixture, through the whole scan, against the oracle's edge rules."""
    for mode in ("zero", "one", "mixed"):
        w, inp = _small_inputs(4, 5, 8, 64, 1, 160, 2, torch.float32, "all", seed=41)
        gm = inp["g"]
        if mode == "zero":
            inp["g"] = torch.zeros_like(gm)
        elif mode == "one":
            inp["g"] = torch.ones_like(gm)
        else:
            r = torch.rand(gm.shape, generator=torch.Generator().manual_seed(42))
            inp["g"] = torch.where(r < 0.3, torch.zeros_like(gm), torch.where(r < 0.6, torch.ones_like(gm), gm))
        cfg, ocfg = _cfgs(w)
        g2 = torch.Generator().manual_seed(43)
        S_in = torch.randn((1, 2, w.M, 64), generator=g2)
        m_in = torch.rand((1, 2, w.M), generator=g2)
        y, S, m = _gpu_scan(cfg, inp, None, S_in, m_in)
        oy, oS, om = _oracle_scan(ocfg, inp, None, S_in, m_in)
        assert _maxabs(y, oy) <= TOL_F32, mode
        assert _maxabs(S, oS) <= TOL_F32, mode
        assert _maxabs(m, om) <= TOL_F32, mode


def test_scan_state_out_aliases_state_in():
    """S_out and m_out may be the same buffers as S_in and m_in."""
    w, inp = _small_inputs(4, 5, 16, 128, 2, 120, 2, torch.bfloat16, "mixed", seed=51)
    cfg, ocfg = _cfgs(w)
    g2 = torch.Generator().manual_seed(52)
    S_in = torch.randn((2, 2, w.M, 128), generator=g2)
    m_in = torch.rand((2, 2, w.M), generator=g2) * 2
    d = _cuda(inp)
    S = S_in.cuda()
    m = m_in.cuda()
    y, _, _ = ramnet.scan_forward(cfg, d["k_logits"], d["q_logits"], d["v"], d["g"], d["z"], cape_mask=d["cape_mask"],
                                  pos0=d["pos0"], S_in=S, m_in=m, S_out=S, m_out=m)
    ramnet.sync_status()
    oy, oS, om = _oracle_scan(ocfg, inp, None, S_in, m_in)
    assert _maxabs(y, oy) <= TOL_BF16 and _maxabs(S, oS) <= TOL_BF16 and _maxabs(m, om) <= TOL_BF16


def test_scan_every_slot_selected():
    """K = M (every slot is written and read by every token) and K = 1."""
    for (d_p, U, K) in [(2, 2, 4), (4, 1, 4), (4, 3, 1)]:
        w, inp = _small_inputs(d_p, U, K, 32, 1, 90, 2, torch.float32, "all", seed=K + d_p)
        cfg, ocfg = _cfgs(w)
        y, S, m = _gpu_scan(cfg, inp)
        oy, oS, om = _oracle_scan(ocfg, inp)
        assert _maxabs(y, oy) <= TOL_F32 and _maxabs(S, oS) <= TOL_F32 and _maxabs(m, om) <= TOL_F32


def test_scan_full_size_is_deterministic():
    """Two calls on the full 340M Top-8 workload give identical bits (y, S, m)."""
    w = WORKLOADS["prefill_340m_top8"]
    cfg, _ = _cfgs(w)
    inp = generate(w, seed=0)
    d = _cuda(inp)
    outs = []
    for _ in range(2):
        outs.append(ramnet.scan_forward(cfg, d["k_logits"], d["q_logits"], d["v"], d["g"], d["z"],
                                        cape_mask=d["cape_mask"], pos0=d["pos0"], out_dtype=torch.bfloat16))
        ramnet.sync_status()
    for a, b2 in zip(outs[0], outs[1]):
        assert torch.equal(a, b2)


@pytest.mark.parametrize("pieces", [1, 3, 7])
def test_scan_from_host_equals_device_scan(pieces):
    """ramnet_scan_forward_host (inputs and y in page-locked host memory, runs along T with the
    state carried and copies overlapping the kernels) gives exactly the device scan's y, S, m."""
    w, inp = _small_inputs(4, 5, 8, 128, 2, 301, 3, torch.bfloat16, "mixed", seed=21)
    cfg, _ = _cfgs(w)
    g = torch.Generator().manual_seed(5)
    S_in = torch.randn((2, 3, w.M, 128), generator=g).cuda()
    m_in = (torch.rand((2, 3, w.M), generator=g) * 2).cuda()
    d = _cuda(inp)
    y, S, m = ramnet.scan_forward(cfg, d["k_logits"], d["q_logits"], d["v"], d["g"], d["z"], cape_mask=d["cape_mask"],
                                  pos0=d["pos0"], S_in=S_in, m_in=m_in, out_dtype=torch.bfloat16)
    host = {k: inp[k].contiguous().pin_memory() for k in ("k_logits", "q_logits", "v", "g", "z")}
    yh = torch.empty(tuple(y.shape), dtype=torch.bfloat16).pin_memory()
    S2 = torch.empty_like(S)
    m2 = torch.empty_like(m)
    scratch = torch.empty(ramnet.scan_forward_host_scratch_bytes(cfg, 2, 301, 3, torch.bfloat16, torch.bfloat16,
                                                                 pieces), dtype=torch.uint8, device="cuda")
    ramnet.scan_forward_host(cfg, host["k_logits"], host["q_logits"], host["v"], host["g"], host["z"], yh, S2, m2,
                             scratch, pieces=pieces, cape_mask=d["cape_mask"], pos0=d["pos0"], S_in=S_in, m_in=m_in)
    torch.cuda.synchronize()
    ramnet.sync_status()
    assert torch.equal(yh, y.cpu())
    assert torch.equal(S2, S) and torch.equal(m2, m)


def test_scan_from_host_fp32_pageable_equals_device_scan():
    """ramnet_scan_forward_host with fp32 inputs and output in ordinary (pageable) host memory,
    no initial state, T not a multiple of the runs: the same bits as the device scan."""
    w, inp = _small_inputs(4, 4, 16, 64, 2, 157, 2, torch.float32, "all", seed=31)
    cfg, _ = _cfgs(w)
    d = _cuda(inp)
    y, S, m = ramnet.scan_forward(cfg, d["k_logits"], d["q_logits"], d["v"], d["g"], d["z"], cape_mask=d["cape_mask"],
                                  pos0=d["pos0"], out_dtype=torch.float32)
    host = {k: inp[k].contiguous() for k in ("k_logits", "q_logits", "v", "g", "z")}
    yh = torch.empty(tuple(y.shape), dtype=torch.float32)
    S2 = torch.empty_like(S)
    m2 = torch.empty_like(m)
    scratch = torch.empty(ramnet.scan_forward_host_scratch_bytes(cfg, 2, 157, 2, torch.float32, torch.float32, 5),
                          dtype=torch.uint8, device="cuda")
    ramnet.scan_forward_host(cfg, host["k_logits"], host["q_logits"], host["v"], host["g"], host["z"], yh, S2, m2,
                             scratch, pieces=5, cape_mask=d["cape_mask"], pos0=d["pos0"])
    torch.cuda.synchronize()
    ramnet.sync_status()
    assert torch.equal(yh, y.cpu())
    assert torch.equal(S2, S) and torch.equal(m2, m)


# ------------------------------------------------------------------ decode step

def _decode_inputs(w: Workload, seed):
    inp = generate(w, seed=seed)
    S0, m0 = generate_decode_state(w, inp["_gen"])
    return inp, S0, m0


def test_decode_step_matches_oracle_over_steps():
    w = WORKLOADS["decode_b256"].with_(B=3, H=4, ring=6)
    cfg, ocfg = _cfgs(w)
    inp, S0, m0 = _decode_inputs(w, seed=11)
    mask = torch.tensor([1, 0, 1, 1], dtype=torch.uint8)
    S, m = S0.cuda(), m0.cuda()
    oS, om = S0.double().numpy().copy(), m0.double().numpy().copy()
    for t in range(w.ring):
        pos = torch.tensor([t, 100 + t, 4095 + t], dtype=torch.int32)
        step = {k: inp[k][:, t].contiguous() for k in ("k_logits", "q_logits", "v", "g", "z")}
        y = ramnet.decode_step(cfg, *(step[k].cuda() for k in ("k_logits", "q_logits", "v", "g", "z")), S, m,
                               pos=pos.cuda(), cape_mask=mask.cuda())
        oy = oracle.decode_step(ocfg, step["k_logits"], step["q_logits"], step["v"], step["g"], step["z"], oS, om,
                                pos=pos, cape_mask=mask)
        ramnet.sync_status()
        assert _maxabs(y, oy) <= TOL_BF16
    assert _maxabs(S, oS) <= TOL_BF16 and _maxabs(m, om) <= TOL_BF16


STEP_SEARCH_CASES = [
    # d_p, U, K, logit mode, renorm -- shapes of the one-warp-per-unit step (K <= 16, d_p <= 8)
    (8, 4, 16, "ties", 1),
    (8, 4, 16, "mixed", 0),
    (4, 5, 8, "ties", 1),
    (3, 4, 5, "mixed", 1),
    (2, 8, 16, "ties", 0),
    (8, 2, 1, "normal", 1),
    (5, 3, 12, "ties", 1),
]


@pytest.mark.parametrize("d_p,U,K,mode,renorm", STEP_SEARCH_CASES)
def test_decode_step_cooperative_search_matches_oracle(d_p, U, K, mode, renorm):
    """Decode steps whose Top-K runs on 16-lane halves of a warp, with tie-heavy and mixed
    logits: a slot chosen wrongly among equal scores writes a different row of S."""
    B, H, steps, d_v = 3, 5, 3, 32
    cfg = ramnet.Config(d_p=d_p, U=U, K=K, d_v=d_v, renorm=renorm)
    ocfg = oracle.OracleConfig(d_p=d_p, U=U, K=K, d_v=d_v, renorm=renorm)
    M = d_p ** U
    g = torch.Generator().manual_seed(d_p * 1000 + K)
    S0 = torch.randn((B, H, M, d_v), generator=g)
    m0 = torch.rand((B, H, M), generator=g) + 0.5
    S, m = S0.cuda(), m0.cuda()
    oS, om = S0.double().numpy().copy(), m0.double().numpy().copy()
    mask = torch.tensor([1, 0, 1, 1, 0], dtype=torch.uint8)
    kl = _logits(B, steps, H, d_p * U, mode, torch.float32, seed=K + 1)
    ql = _logits(B, steps, H, d_p * U, mode, torch.float32, seed=K + 2)
    for t in range(steps):
        v = torch.randn((B, H, d_v), generator=g)
        z = torch.sigmoid(torch.randn((B, H, d_v), generator=g))
        gt = torch.sigmoid(torch.randn((B, H), generator=g))
        pos = torch.tensor([t, 77 + t, M + 5 + t], dtype=torch.int32)
        k_t, q_t = kl[:, t].contiguous(), ql[:, t].contiguous()
        y = ramnet.decode_step(cfg, k_t.cuda(), q_t.cuda(), v.cuda(), gt.cuda(), z.cuda(), S, m, pos=pos.cuda(),
                               cape_mask=mask.cuda(), out_dtype=torch.float32)
        oy = oracle.decode_step(ocfg, k_t, q_t, v, gt, z, oS, om, pos=pos, cape_mask=mask)
        ramnet.sync_status()
        assert _maxabs(y, oy) <= TOL_F32
    assert _maxabs(S, oS) <= TOL_F32 and _maxabs(m, om) <= TOL_F32


STEP_PERSISTENT_CASES = [
    # d_p, U, K, logit mode, renorm, d_v -- shapes served by the persistent decode-step kernel
    (4, 5, 32, "ties", 1, 128),
    (4, 5, 32, "mixed", 0, 64),
    (16, 2, 8, "normal", 1, 128),
    (3, 5, 64, "ties", 1, 32),
    (16, 3, 20, "mixed", 1, 16),
]


@pytest.mark.parametrize("d_p,U,K,mode,renorm,d_v", STEP_PERSISTENT_CASES)
def test_decode_step_persistent_kernel_matches_oracle(d_p, U, K, mode, renorm, d_v):
    """Decode steps with K > 16 or d_p > 8, which run the persistent kernel (decoder warps with
    the one-thread search, row warps per unit), against the oracle over three steps."""
    B, H, steps = 3, 4, 3
    cfg = ramnet.Config(d_p=d_p, U=U, K=K, d_v=d_v, renorm=renorm)
    ocfg = oracle.OracleConfig(d_p=d_p, U=U, K=K, d_v=d_v, renorm=renorm)
    M = d_p ** U
    g = torch.Generator().manual_seed(d_p * 100 + K)
    S0 = torch.randn((B, H, M, d_v), generator=g)
    m0 = torch.rand((B, H, M), generator=g) + 0.5
    S, m = S0.cuda(), m0.cuda()
    oS, om = S0.double().numpy().copy(), m0.double().numpy().copy()
    mask = torch.tensor([1, 1, 0, 1], dtype=torch.uint8)
    kl = _logits(B, steps, H, d_p * U, mode, torch.bfloat16, seed=K + 3)
    ql = _logits(B, steps, H, d_p * U, mode, torch.bfloat16, seed=K + 4)
    for t in range(steps):
        v = torch.randn((B, H, d_v), generator=g).to(torch.bfloat16)
        z = torch.sigmoid(torch.randn((B, H, d_v), generator=g)).to(torch.bfloat16)
        gt = torch.sigmoid(torch.randn((B, H), generator=g)).to(torch.bfloat16)
        pos = torch.tensor([t, 9 + t, 2 * M + t], dtype=torch.int32)
        k_t, q_t = kl[:, t].contiguous(), ql[:, t].contiguous()
        y = ramnet.decode_step(cfg, k_t.cuda(), q_t.cuda(), v.cuda(), gt.cuda(), z.cuda(), S, m, pos=pos.cuda(),
                               cape_mask=mask.cuda(), out_dtype=torch.float32)
        oy = oracle.decode_step(ocfg, k_t, q_t, v, gt, z, oS, om, pos=pos, cape_mask=mask)
        ramnet.sync_status()
        assert _maxabs(y, oy) <= TOL_BF16
    assert _maxabs(S, oS) <= TOL_BF16 and _maxabs(m, om) <= TOL_BF16


def test_decode_step_full_size_sampled_units():
    """One step of the full batched decode workload (state resident in HBM); sampled
    (b,h) units are recomputed by the oracle from their pre-step state."""
    w = WORKLOADS["decode_b256"]
    cfg, ocfg = _cfgs(w)
    inp = generate(w, seed=0)
    gen = torch.Generator(device="cuda").manual_seed(1)
    S = torch.randn((w.B, w.H, w.M, w.d_v), device="cuda", generator=gen)
    m = torch.rand((w.B, w.H, w.M), device="cuda", generator=gen) * 1.5 + 0.5
    units = [(0, 0), (17, 5), (w.B - 1, w.H - 1)]
    before = {u: (S[u].double().cpu().numpy().copy(), m[u].double().cpu().numpy().copy()) for u in units}
    pos = torch.arange(w.B, dtype=torch.int32) * 7
    step = {k: inp[k][:, 3].contiguous() for k in ("k_logits", "q_logits", "v", "g", "z")}
    y = ramnet.decode_step(cfg, *(step[k].cuda() for k in ("k_logits", "q_logits", "v", "g", "z")), S, m,
                           pos=pos.cuda(), cape_mask=inp["cape_mask"].cuda())
    ramnet.sync_status()
    for (b, h) in units:
        Sb = before[(b, h)][0][None, None].copy()
        mb = before[(b, h)][1][None, None].copy()
        sl = {k: step[k][b:b + 1, h:h + 1] for k in step}
        oy = oracle.decode_step(ocfg, sl["k_logits"], sl["q_logits"], sl["v"], sl["g"], sl["z"], Sb, mb,
                                pos=pos[b:b + 1], cape_mask=inp["cape_mask"][h:h + 1])
        assert _maxabs(y[b, h], oy[0, 0]) <= TOL_BF16
        assert _maxabs(S[b, h], Sb[0, 0]) <= TOL_BF16
        assert _maxabs(m[b, h], mb[0, 0]) <= TOL_BF16


def test_decode_step_chain_equals_scan():
    """T single decode steps equal one prefill scan of the same T tokens."""
    w, inp = _small_inputs(4, 5, 8, 64, 2, 40, 2, torch.float32, "mixed", seed=12)
    cfg, _ = _cfgs(w)
    y, S, m = _gpu_scan(cfg, inp)
    Sd = torch.zeros((2, 2, w.M, 64), device="cuda")
    md = torch.zeros((2, 2, w.M), device="cuda")
    d = _cuda(inp)
    for t in range(40):
        yd = ramnet.decode_step(cfg, d["k_logits"][:, t].contiguous(), d["q_logits"][:, t].contiguous(),
                                d["v"][:, t].contiguous(), d["g"][:, t].contiguous(), d["z"][:, t].contiguous(),
                                Sd, md, pos=d["pos0"] + t, cape_mask=d["cape_mask"])
        assert _maxabs(yd, y[:, t]) <= TOL_F32
    assert _maxabs(Sd, S) <= TOL_F32 and _maxabs(md, m) <= TOL_F32
