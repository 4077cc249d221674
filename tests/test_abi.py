"""The C-ABI library: it loads, exports every symbol include/ramnet.h declares, and its
host-side argument checks reject bad calls before anything is launched (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from sparse_slot_recurrent_b200 import build as build_mod
from sparse_slot_recurrent_b200 import ramnet

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ramnet.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return ramnet.load()


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(ramnet_\w+)\s*\(", src, re.M)))


def test_header_declares_the_entry_points():
    names = _declared()
    assert set(names) == set(ramnet.EXPORTED), names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", build_mod.OUT], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in _declared():
        assert name in exported, name
        assert hasattr(lib, name)


def _cfg(**kw):
    base = dict(d_p=4, U=5, K=8, d_v=128)
    base.update(kw)
    return ramnet.Config(**base)


FAKE = 1 << 40  # 16-byte aligned, never dereferenced: every call below fails host-side


def _decode(lib, cfg, B=1, T=4, H=1, logits=FAKE, dt=ramnet.RAMNET_BF16, idx=FAKE, w=FAKE, pos0=None, strides=None):
    c = cfg._c()
    st = None if strides is None else ctypes.byref(ramnet._Strides(*strides))
    return lib.ramnet_decode_addresses(ctypes.byref(c), B, T, H, logits, dt, st, pos0, None, idx, w, None)


@pytest.mark.parametrize("kw", [dict(d_p=1), dict(d_p=17), dict(U=0), dict(U=9), dict(d_p=16, U=5),
                                dict(K=0), dict(K=65), dict(d_p=2, U=2, K=5), dict(d_v=48), dict(d_v=512),
                                dict(eps_gsu=-1.0), dict(eps_norm=float("nan"))])
def test_bad_config_rejected(lib, kw):
    assert _decode(lib, _cfg(**kw)) == ramnet.RAMNET_ERR_INVALID_ARG
    assert ramnet.last_error() != ""


def test_bad_pointers_and_sizes_rejected(lib):
    cfg = _cfg()
    assert _decode(lib, cfg, logits=None) == ramnet.RAMNET_ERR_INVALID_ARG
    assert "logits" in ramnet.last_error()
    assert _decode(lib, cfg, logits=FAKE + 1) == ramnet.RAMNET_ERR_INVALID_ARG
    assert "aligned" in ramnet.last_error()
    assert _decode(lib, cfg, logits=FAKE + 2, dt=ramnet.RAMNET_F32) == ramnet.RAMNET_ERR_INVALID_ARG
    assert _decode(lib, cfg, strides=(80, -20, 20)) == ramnet.RAMNET_ERR_INVALID_ARG
    assert "stride" in ramnet.last_error()
    assert _decode(lib, cfg, idx=FAKE + 4) == ramnet.RAMNET_ERR_INVALID_ARG
    assert _decode(lib, cfg, idx=None) == ramnet.RAMNET_ERR_INVALID_ARG
    assert _decode(lib, cfg, pos0=FAKE + 8) == ramnet.RAMNET_ERR_INVALID_ARG
    assert _decode(lib, cfg, B=0) == ramnet.RAMNET_ERR_INVALID_ARG
    assert _decode(lib, cfg, T=-3) == ramnet.RAMNET_ERR_INVALID_ARG
    assert _decode(lib, cfg, dt=7) == ramnet.RAMNET_ERR_INVALID_ARG


def _scan(lib, cfg, B=2, T=8, H=2, ws_bytes=None, S_in=None, y=FAKE, ws=FAKE):
    c = cfg._c()
    if ws_bytes is None:
        ws_bytes = lib.ramnet_scan_workspace_bytes(ctypes.byref(c), B, T, H)
    return lib.ramnet_scan_forward(ctypes.byref(c), B, T, H, ramnet.RAMNET_BF16, FAKE, FAKE, FAKE, FAKE, FAKE,
                                   None, None, None, S_in, None, y, ramnet.RAMNET_F32, FAKE, FAKE, ws, ws_bytes,
                                   None)


def test_scan_workspace_size(lib):
    cfg = _cfg()
    c = cfg._c()
    need = lib.ramnet_scan_workspace_bytes(ctypes.byref(c), 8, 4096, 8)
    assert need >= 4 * 8 * 4096 * 8 * 8 * 4
    bad = _cfg(d_p=1)._c()
    assert lib.ramnet_scan_workspace_bytes(ctypes.byref(bad), 8, 4096, 8) == 0
    assert _scan(lib, cfg, ws_bytes=16) == ramnet.RAMNET_ERR_INVALID_ARG
    assert "workspace" in ramnet.last_error()
    assert _scan(lib, cfg, ws=None) == ramnet.RAMNET_ERR_INVALID_ARG
    assert _scan(lib, cfg, y=None) == ramnet.RAMNET_ERR_INVALID_ARG
    assert _scan(lib, cfg, S_in=FAKE + 4) == ramnet.RAMNET_ERR_INVALID_ARG


def test_scan_rejects_slot_arrays_beyond_tensor_memory(lib):
    # M = 65536 slots x 256 channels x 4 B = 64 MiB per head: far beyond 8 SMs of TMEM
    cfg = _cfg(d_p=16, U=4, K=8, d_v=256)
    assert _scan(lib, cfg) == ramnet.RAMNET_ERR_UNSUPPORTED
    assert "tensor memory" in ramnet.last_error()


def test_decode_step_checks(lib):
    cfg = _cfg(d_p=8, U=4, K=16)
    c = cfg._c()
    args = [ctypes.byref(c), 4, 2, ramnet.RAMNET_BF16, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE, FAKE,
            FAKE, ramnet.RAMNET_F32, None]
    bad = list(args)
    bad[12] = None  # S
    assert lib.ramnet_decode_step(*bad) == ramnet.RAMNET_ERR_INVALID_ARG
    bad = list(args)
    bad[1] = 0
    assert lib.ramnet_decode_step(*bad) == ramnet.RAMNET_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="only meaningful without a CUDA device")
def test_valid_call_without_device_reports_cuda_error(lib):
    # arguments pass every host check; with no device the first CUDA call fails cleanly
    assert _decode(lib, _cfg()) == ramnet.RAMNET_ERR_CUDA
    assert ramnet.last_error() != ""


def test_scan_workspace_is_events_then_headers(lib):
    # decoded events (16 bytes each, 2*K per token, grouped in chunks of C tokens), then one
    # header per (head, chunk, rank) at a 256-byte boundary; the larger of the two input
    # dtypes' plans
    for (d_p, U, K, d_v), (B, T, H) in [((4, 5, 8, 128), (8, 4096, 8)), ((3, 5, 7, 32), (1, 77, 2)),
                                         ((16, 2, 64, 256), (2, 33, 3)), ((4, 5, 32, 128), (8, 8192, 8))]:
        cfg = _cfg(d_p=d_p, U=U, K=K, d_v=d_v)
        c = cfg._c()
        want = 0
        for dt in (torch.bfloat16, torch.float32):
            lay = ramnet.scan_layout(cfg, dt)
            assert lay.chunk >= 1 and lay.chunk & (lay.chunk - 1) == 0 and 64 % lay.chunk == 0
            assert lay.ncta in (1, 2, 4, 8) and lay.scan_warps == 16 and lay.hdr_words % 4 == 0
            assert lay.hdr_words >= 4 + lay.scan_warps + 1 + (lay.chunk + 3) // 4
            nch = -(-T // lay.chunk)
            events = B * H * nch * 2 * lay.chunk * K * 16
            want = max(want, (events + 255) // 256 * 256 + B * H * nch * lay.ncta * lay.hdr_words * 4)
        assert lib.ramnet_scan_workspace_bytes(ctypes.byref(c), B, T, H) == want


def test_scan_layout_checks(lib):
    c = _cfg()._c()
    out = [ctypes.c_int32() for _ in range(4)]
    assert lib.ramnet_scan_layout(ctypes.byref(c), 9, *(ctypes.byref(v) for v in out)) == ramnet.RAMNET_ERR_INVALID_ARG
    assert lib.ramnet_scan_layout(ctypes.byref(c), ramnet.RAMNET_BF16, None, *(ctypes.byref(v) for v in out[1:])) == \
        ramnet.RAMNET_ERR_INVALID_ARG
    big = _cfg(d_p=16, U=4, K=8, d_v=256)._c()
    assert lib.ramnet_scan_layout(ctypes.byref(big), ramnet.RAMNET_BF16, *(ctypes.byref(v) for v in out)) == \
        ramnet.RAMNET_ERR_UNSUPPORTED


def test_two_launch_form_checks(lib):
    cfg = _cfg()
    c = cfg._c()
    B, T, H = 2, 8, 2
    need = lib.ramnet_scan_workspace_bytes(ctypes.byref(c), B, T, H)
    route = lambda k=FAKE, ws=FAKE, n=need: lib.ramnet_scan_route(
        ctypes.byref(c), B, T, H, ramnet.RAMNET_BF16, k, FAKE, FAKE, None, None, ws, n, None)
    recur = lambda v=FAKE, ws=FAKE, n=need, od=ramnet.RAMNET_F32: lib.ramnet_scan_recur(
        ctypes.byref(c), B, T, H, ramnet.RAMNET_BF16, v, FAKE, None, None, None, FAKE, od, FAKE, FAKE, ws, n, None)
    assert route(k=None) == ramnet.RAMNET_ERR_INVALID_ARG and "k_logits" in ramnet.last_error()
    assert route(n=need - 1) == ramnet.RAMNET_ERR_INVALID_ARG and "workspace" in ramnet.last_error()
    assert route(ws=FAKE + 8) == ramnet.RAMNET_ERR_INVALID_ARG and "aligned" in ramnet.last_error()
    assert recur(v=None) == ramnet.RAMNET_ERR_INVALID_ARG and "v" in ramnet.last_error()
    assert recur(od=5) == ramnet.RAMNET_ERR_INVALID_ARG
    assert recur(ws=None) == ramnet.RAMNET_ERR_INVALID_ARG


def test_scan_from_host_checks(lib):
    cfg = _cfg()
    c = cfg._c()
    B, T, H = 2, 40, 2
    need = lib.ramnet_scan_forward_host_scratch_bytes(ctypes.byref(c), B, T, H, ramnet.RAMNET_BF16,
                                                      ramnet.RAMNET_BF16, 3)
    assert need > lib.ramnet_scan_workspace_bytes(ctypes.byref(c), B, (T + 2) // 3, H)
    assert lib.ramnet_scan_forward_host_scratch_bytes(ctypes.byref(c), B, T, H, 7, ramnet.RAMNET_BF16, 3) == 0

    def call(pieces=3, scratch_bytes=need, k=FAKE, y=FAKE, scratch=FAKE):
        return lib.ramnet_scan_forward_host(ctypes.byref(c), B, T, H, ramnet.RAMNET_BF16, k, FAKE, FAKE, FAKE, FAKE,
                                            None, None, None, None, None, y, ramnet.RAMNET_BF16, FAKE, FAKE, pieces,
                                            scratch, scratch_bytes, None)

    assert call(pieces=0) == ramnet.RAMNET_ERR_INVALID_ARG
    assert "pieces" in ramnet.last_error()
    assert call(scratch_bytes=need - 1) == ramnet.RAMNET_ERR_INVALID_ARG
    assert "scratch" in ramnet.last_error()
    assert call(k=None) == ramnet.RAMNET_ERR_INVALID_ARG
    assert call(y=None) == ramnet.RAMNET_ERR_INVALID_ARG
    assert call(scratch=FAKE + 4) == ramnet.RAMNET_ERR_INVALID_ARG
