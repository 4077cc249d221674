"""ramnet_scan_forward_noalloc (the prefill scan on the library's built-in scratch) against
ramnet_scan_forward with a caller workspace, both through the C ABI.

Two calls in a row on the built-in scratch must each match the workspace call within the
parity tolerance (max-abs 1e-5 for fp32 inputs, 1e-3 for bf16 inputs); sizes whose
scratch exceeds the built-in array must be refused with RAMNET_ERR_UNSUPPORTED.  The file
name sorts last so that it also runs after every other GPU test.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_slot_recurrent_b200 import ramnet
from sparse_slot_recurrent_b200.workloads import Workload, generate, generate_decode_state

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    ramnet.load()
    yield
    ramnet.sync_status()


CASES = [
    # B, H, T, d_p, U, K, d_v, in dtype, with initial state
    (1, 2, 300, 4, 5, 8, 16, torch.float32, False),
    (2, 2, 257, 4, 4, 16, 64, torch.bfloat16, True),
    (1, 1, 97, 8, 4, 16, 128, torch.bfloat16, True),
]


def _maxabs(a, b):
    return float((a.double() - b.double()).abs().max().cpu()) if a.numel() else 0.0


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}H{c[1]}T{c[2]}dp{c[3]}U{c[4]}K{c[5]}dv{c[6]}" for c in CASES])
def test_noalloc_matches_workspace_call_twice(case):
    B, H, T, d_p, U, K, d_v, dt, with_state = case
    w = Workload("noalloc", B=B, H=H, T=T, d_p=d_p, U=U, K=K, d_v=d_v, in_dtype=dt, cape=True, logit_std=1.5)
    cfg = ramnet.Config(d_p=d_p, U=U, K=K, d_v=d_v)
    assert 0 < ramnet.scan_workspace_bytes(cfg, B, T, H) <= ramnet.NOALLOC_SCRATCH_BYTES
    gen = torch.Generator(device="cuda")
    gen.manual_seed(11)
    inp = generate(w, seed=5, device="cuda")
    S_in = m_in = None
    if with_state:
        S_in, m_in = generate_decode_state(w, gen, device="cuda")
    norm_w = torch.rand(d_v, generator=gen, device="cuda") + 0.5
    args = (inp["k_logits"], inp["q_logits"], inp["v"], inp["g"], inp["z"])
    kw = dict(norm_w=norm_w, cape_mask=inp["cape_mask"], pos0=inp["pos0"], S_in=S_in, m_in=m_in)
    y_ref, S_ref, m_ref = ramnet.scan_forward(cfg, *args, out_dtype=torch.float32, **kw)
    tol = 1e-5 if dt == torch.float32 else 1e-3
    for _ in range(2):
        y = torch.full_like(y_ref, float("nan"))
        S = torch.full_like(S_ref, float("nan"))
        m = torch.full_like(m_ref, float("nan"))
        ramnet.scan_forward_noalloc(cfg, *args, y, S, m, **kw)
        ramnet.sync_status()
        assert torch.isfinite(y).all() and torch.isfinite(S).all() and torch.isfinite(m).all()
        assert _maxabs(y, y_ref) <= tol
        assert _maxabs(S, S_ref) <= tol
        assert _maxabs(m, m_ref) <= tol


def test_noalloc_refuses_sizes_beyond_the_static_scratch():
    cfg = ramnet.Config(d_p=4, U=5, K=32, d_v=128)
    B, T, H = 8, 8192, 8
    need = ramnet.scan_workspace_bytes(cfg, B, T, H)
    assert need > ramnet.NOALLOC_SCRATCH_BYTES
    lib = ramnet.load()
    c = cfg._c()
    st = lib.ramnet_scan_forward_noalloc(ctypes.byref(c), B, T, H, ramnet.RAMNET_BF16, *([None] * 10), None,
                                         ramnet.RAMNET_F32, None, None, None)
    assert st == ramnet.RAMNET_ERR_UNSUPPORTED
    msg = ramnet.last_error()
    assert str(need) in msg and str(ramnet.NOALLOC_SCRATCH_BYTES) in msg
    np.testing.assert_equal(lib.ramnet_sync_status(None), ramnet.RAMNET_OK)
