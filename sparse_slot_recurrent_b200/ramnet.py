"""Thin Python binding of the RAM-Net C ABI (``include/ramnet.h``).

Argument marshalling only: torch supplies device memory and the current CUDA stream;
every step of the layer runs in the library's kernels.  The library is loaded from the
package directory (``libramnet.so``, built by ``build.py``; with the environment variable
RAMNET_DEBUG=1 the range-checking build ``libramnet_debug.so``); if it is missing or fails
to load, every call raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
DEBUG = os.environ.get("RAMNET_DEBUG", "0") not in ("", "0")
LIB_PATH = os.path.join(_PKG, "libramnet_debug.so" if DEBUG else "libramnet.so")

RAMNET_OK, RAMNET_ERR_INVALID_ARG, RAMNET_ERR_UNSUPPORTED, RAMNET_ERR_CUDA, RAMNET_ERR_TIMEOUT, \
    RAMNET_ERR_DEVICE_CHECK = range(6)
RAMNET_F32, RAMNET_BF16 = 0, 1

# every symbol include/ramnet.h declares
EXPORTED = ("ramnet_decode_addresses", "ramnet_scan_workspace_bytes", "ramnet_scan_layout", "ramnet_scan_forward",
            "ramnet_scan_route", "ramnet_scan_recur", "ramnet_scan_forward_noalloc", "ramnet_decode_step",
            "ramnet_scan_forward_host_scratch_bytes", "ramnet_scan_forward_host",
            "ramnet_selftest_wait_timeout", "ramnet_set_scan_wait_limit", "ramnet_sync_status", "ramnet_last_error")
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024  # RAMNET_NOALLOC_SCRATCH_BYTES


class RamnetError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"ramnet status {status}: {msg}")
        self.status = status


class _Strides(ctypes.Structure):
    _fields_ = [("b", ctypes.c_int64), ("t", ctypes.c_int64), ("h", ctypes.c_int64)]


class _Cfg(ctypes.Structure):
    _fields_ = [("d_p", ctypes.c_int32), ("U", ctypes.c_int32), ("K", ctypes.c_int32),
                ("d_v", ctypes.c_int32), ("eps_gsu", ctypes.c_float),
                ("eps_norm", ctypes.c_float), ("renorm", ctypes.c_int32)]


@dataclass(frozen=True)
class Config:
    d_p: int
    U: int
    K: int
    d_v: int
    eps_gsu: float = 1e-6
    eps_norm: float = 1e-6
    renorm: int = 1

    @property
    def M(self) -> int:
        return self.d_p ** self.U

    @property
    def L(self) -> int:
        return self.d_p * self.U

    def _c(self) -> _Cfg:
        return _Cfg(self.d_p, self.U, self.K, self.d_v, self.eps_gsu, self.eps_norm, self.renorm)


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int32


def load() -> ctypes.CDLL:
    """Load libramnet.so (raises if it is absent or lacks a declared symbol)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with sparse_slot_recurrent_b200/build.py"
                           + (" --debug" if DEBUG else ""))
    lib = ctypes.CDLL(LIB_PATH)
    for name in EXPORTED:
        if not hasattr(lib, name):
            raise RuntimeError(f"{LIB_PATH} does not export {name}")
    C = ctypes.POINTER(_Cfg)
    lib.ramnet_decode_addresses.restype = ctypes.c_int
    lib.ramnet_decode_addresses.argtypes = [C, _I, _I, _I, _P, ctypes.c_int, ctypes.POINTER(_Strides), _P, _P, _P,
                                            _P, _P]
    lib.ramnet_scan_workspace_bytes.restype = ctypes.c_size_t
    lib.ramnet_scan_workspace_bytes.argtypes = [C, _I, _I, _I]
    lib.ramnet_scan_layout.restype = ctypes.c_int
    lib.ramnet_scan_layout.argtypes = [C, ctypes.c_int, _P, _P, _P, _P]
    lib.ramnet_scan_forward.restype = ctypes.c_int
    lib.ramnet_scan_forward.argtypes = [C, _I, _I, _I, ctypes.c_int, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                        _P, ctypes.c_int, _P, _P, _P, ctypes.c_size_t, _P]
    lib.ramnet_scan_route.restype = ctypes.c_int
    lib.ramnet_scan_route.argtypes = [C, _I, _I, _I, ctypes.c_int, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
    lib.ramnet_scan_recur.restype = ctypes.c_int
    lib.ramnet_scan_recur.argtypes = [C, _I, _I, _I, ctypes.c_int, _P, _P, _P, _P, _P, _P, ctypes.c_int, _P, _P,
                                      _P, ctypes.c_size_t, _P]
    lib.ramnet_scan_forward_noalloc.restype = ctypes.c_int
    lib.ramnet_scan_forward_noalloc.argtypes = [C, _I, _I, _I, ctypes.c_int, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                                _P, _P, ctypes.c_int, _P, _P, _P]
    lib.ramnet_decode_step.restype = ctypes.c_int
    lib.ramnet_decode_step.argtypes = [C, _I, _I, ctypes.c_int, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                       ctypes.c_int, _P]
    lib.ramnet_selftest_wait_timeout.restype = ctypes.c_int
    lib.ramnet_selftest_wait_timeout.argtypes = [ctypes.c_uint32, _P]
    lib.ramnet_scan_forward_host_scratch_bytes.restype = ctypes.c_size_t
    lib.ramnet_scan_forward_host_scratch_bytes.argtypes = [_P, _I, _I, _I, _I, _I, _I]
    lib.ramnet_scan_forward_host.restype = ctypes.c_int
    lib.ramnet_scan_forward_host.argtypes = ([_P, _I, _I, _I, _I] + [_P] * 11 + [_I] + [_P] * 2 +
                                             [_I, _P, ctypes.c_size_t, _P])
    lib.ramnet_set_scan_wait_limit.restype = ctypes.c_int
    lib.ramnet_set_scan_wait_limit.argtypes = [ctypes.c_uint32]
    lib.ramnet_sync_status.restype = ctypes.c_int
    lib.ramnet_sync_status.argtypes = [_P]
    lib.ramnet_last_error.restype = ctypes.c_char_p
    lib.ramnet_last_error.argtypes = []
    _lib = lib
    return lib


def last_error() -> str:
    return load().ramnet_last_error().decode()


def _check(status: int):
    if status != RAMNET_OK:
        raise RamnetError(status, last_error())


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _dt(t) -> int:
    if t.dtype == torch.bfloat16:
        return RAMNET_BF16
    if t.dtype == torch.float32:
        return RAMNET_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dense(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def decode_addresses(cfg: Config, logits: torch.Tensor, pos0=None, cape_mask=None, idx_out=None, w_out=None,
                     stream=None):
    """logits [B,T,H,U*d_p] (fp32 or bf16; any strides with the last dimension contiguous)
    -> (idx int32 [B,T,H,K], w fp32 [B,T,H,K])."""
    B, T, H, L = logits.shape
    if logits.stride(-1) != 1:
        raise ValueError("the last dimension of logits must be contiguous")
    _dense(pos0, cape_mask)
    if idx_out is None:
        idx_out = torch.empty((B, T, H, cfg.K), dtype=torch.int32, device=logits.device)
    if w_out is None:
        w_out = torch.empty((B, T, H, cfg.K), dtype=torch.float32, device=logits.device)
    c = cfg._c()
    st = _Strides(*logits.stride()[:3])
    _check(load().ramnet_decode_addresses(ctypes.byref(c), B, T, H, _ptr(logits), _dt(logits), ctypes.byref(st),
                                          _ptr(pos0), _ptr(cape_mask), _ptr(idx_out), _ptr(w_out), _stream(stream)))
    return idx_out, w_out


def scan_workspace_bytes(cfg: Config, B: int, T: int, H: int) -> int:
    c = cfg._c()
    return int(load().ramnet_scan_workspace_bytes(ctypes.byref(c), B, T, H))


@dataclass(frozen=True)
class ScanLayout:
    chunk: int
    ncta: int
    scan_warps: int
    hdr_words: int


def scan_layout(cfg: Config, in_dtype=torch.bfloat16) -> ScanLayout:
    """The prefill's work split for this config and input dtype (see ramnet_scan_layout)."""
    vals = [ctypes.c_int32() for _ in range(4)]
    c = cfg._c()
    dt = RAMNET_BF16 if in_dtype == torch.bfloat16 else RAMNET_F32
    _check(load().ramnet_scan_layout(ctypes.byref(c), dt, *(ctypes.byref(v) for v in vals)))
    return ScanLayout(*(v.value for v in vals))


def scan_forward(cfg: Config, k_logits, q_logits, v, g, z, norm_w=None, cape_mask=None, pos0=None, S_in=None,
                 m_in=None, out_dtype=torch.float32, y=None, S_out=None, m_out=None, workspace=None, stream=None):
    """Prefill scan.  Returns (y [B,T,H,d_v], S_out [B,H,M,d_v], m_out [B,H,M])."""
    B, T, H, L = k_logits.shape
    dev = k_logits.device
    _dense(k_logits, q_logits, v, g, z, norm_w, cape_mask, pos0, S_in, m_in)
    if y is None:
        y = torch.empty((B, T, H, cfg.d_v), dtype=out_dtype, device=dev)
    if S_out is None:
        S_out = torch.empty((B, H, cfg.M, cfg.d_v), dtype=torch.float32, device=dev)
    if m_out is None:
        m_out = torch.empty((B, H, cfg.M), dtype=torch.float32, device=dev)
    need = scan_workspace_bytes(cfg, B, T, H)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    c = cfg._c()
    _check(load().ramnet_scan_forward(
        ctypes.byref(c), B, T, H, _dt(k_logits), _ptr(k_logits), _ptr(q_logits), _ptr(v), _ptr(g), _ptr(z),
        _ptr(norm_w), _ptr(cape_mask), _ptr(pos0), _ptr(S_in), _ptr(m_in), _ptr(y), _dt(y), _ptr(S_out),
        _ptr(m_out), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return y, S_out, m_out


def scan_forward_host_scratch_bytes(cfg: Config, B: int, T: int, H: int, in_dtype, out_dtype, pieces: int) -> int:
    c = cfg._c()
    codes = {torch.bfloat16: RAMNET_BF16, torch.float32: RAMNET_F32}
    n = load().ramnet_scan_forward_host_scratch_bytes(ctypes.byref(c), B, T, H, codes[in_dtype], codes[out_dtype],
                                                      pieces)
    if n == 0:
        raise RamnetError(RAMNET_ERR_INVALID_ARG, last_error() or "bad sizes")
    return n


def scan_forward_host(cfg: Config, k_logits, q_logits, v, g, z, y, S_out, m_out, scratch, pieces=4, norm_w=None,
                      cape_mask=None, pos0=None, S_in=None, m_in=None, stream=None):
    """Prefill scan with k_logits, q_logits, v, g, z and y in host memory (CPU tensors, page-locked
    for overlap) and the rest on the device; run in ``pieces`` runs along T whose copies overlap
    the kernels.  ``scratch`` is a uint8 device tensor of scan_forward_host_scratch_bytes()."""
    B, T, H, L = k_logits.shape
    for t in (k_logits, q_logits, v, g, z, y):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("host tensors must be contiguous CPU tensors")
    _dense(norm_w, cape_mask, pos0, S_in, m_in, S_out, m_out, scratch)
    c = cfg._c()
    _check(load().ramnet_scan_forward_host(
        ctypes.byref(c), B, T, H, _dt(k_logits), k_logits.data_ptr(), q_logits.data_ptr(), v.data_ptr(), g.data_ptr(),
        z.data_ptr(), _ptr(norm_w), _ptr(cape_mask), _ptr(pos0), _ptr(S_in), _ptr(m_in), y.data_ptr(), _dt(y),
        _ptr(S_out), _ptr(m_out), pieces, _ptr(scratch), scratch.numel() * scratch.element_size(), _stream(stream)))
    return y, S_out, m_out


def scan_route(cfg: Config, k_logits, q_logits, g, workspace, cape_mask=None, pos0=None, stream=None):
    """First launch of scan_forward: address decode, CAPE, write retentions, event grouping
    into ``workspace`` (uint8 device tensor of at least scan_workspace_bytes())."""
    B, T, H, L = k_logits.shape
    _dense(k_logits, q_logits, g, cape_mask, pos0, workspace)
    c = cfg._c()
    _check(load().ramnet_scan_route(ctypes.byref(c), B, T, H, _dt(k_logits), _ptr(k_logits), _ptr(q_logits), _ptr(g),
                                    _ptr(cape_mask), _ptr(pos0), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)))


def scan_recur(cfg: Config, v, z, y, S_out, m_out, workspace, norm_w=None, S_in=None, m_in=None, stream=None):
    """Second launch of scan_forward: the recurrence over the events scan_route wrote."""
    B, T, H, dv = v.shape
    _dense(v, z, y, S_out, m_out, workspace, norm_w, S_in, m_in)
    c = cfg._c()
    _check(load().ramnet_scan_recur(ctypes.byref(c), B, T, H, _dt(v), _ptr(v), _ptr(z), _ptr(norm_w), _ptr(S_in),
                                    _ptr(m_in), _ptr(y), _dt(y), _ptr(S_out), _ptr(m_out), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)))
    return y, S_out, m_out


def scan_forward_noalloc(cfg: Config, k_logits, q_logits, v, g, z, y, S_out, m_out, norm_w=None, cape_mask=None,
                         pos0=None, S_in=None, m_in=None, stream=None):
    """Prefill scan on the library's built-in scratch (no workspace argument).  All outputs
    are passed in; nothing is allocated.  Returns (y, S_out, m_out)."""
    B, T, H, L = k_logits.shape
    _dense(k_logits, q_logits, v, g, z, norm_w, cape_mask, pos0, S_in, m_in, y, S_out, m_out)
    c = cfg._c()
    _check(load().ramnet_scan_forward_noalloc(
        ctypes.byref(c), B, T, H, _dt(k_logits), _ptr(k_logits), _ptr(q_logits), _ptr(v), _ptr(g), _ptr(z),
        _ptr(norm_w), _ptr(cape_mask), _ptr(pos0), _ptr(S_in), _ptr(m_in), _ptr(y), _dt(y), _ptr(S_out),
        _ptr(m_out), _stream(stream)))
    return y, S_out, m_out


def decode_step(cfg: Config, k_logits, q_logits, v, g, z, S, m, pos=None, norm_w=None, cape_mask=None,
                out_dtype=torch.float32, y=None, stream=None):
    """One decode token per (b,h); S [B,H,M,d_v] and m [B,H,M] fp32 are updated in place.
    Returns y [B,H,d_v]."""
    B, H, L = k_logits.shape
    _dense(k_logits, q_logits, v, g, z, S, m, pos, norm_w, cape_mask)
    if y is None:
        y = torch.empty((B, H, cfg.d_v), dtype=out_dtype, device=k_logits.device)
    c = cfg._c()
    _check(load().ramnet_decode_step(ctypes.byref(c), B, H, _dt(k_logits), _ptr(k_logits), _ptr(q_logits), _ptr(v),
                                     _ptr(g), _ptr(z), _ptr(norm_w), _ptr(cape_mask), _ptr(pos), _ptr(S), _ptr(m),
                                     _ptr(y), _dt(y), _stream(stream)))
    return y


def selftest_wait_timeout(limit_us: int, stream=None):
    """Launch the failure-detection self-test (a bounded wait that must run out)."""
    _check(load().ramnet_selftest_wait_timeout(limit_us, _stream(stream)))


def set_scan_wait_limit(limit_us: int):
    """Limit of the prefill recurrence's bounded waits for later launches (0: 2 s default)."""
    _check(load().ramnet_set_scan_wait_limit(limit_us))


def sync_status(stream=None):
    """Wait for the stream and raise if a kernel recorded a timeout or failed check."""
    _check(load().ramnet_sync_status(_stream(stream)))
