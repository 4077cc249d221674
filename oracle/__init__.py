"""CPU oracle for the RAM-Net layer core.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library never
calls it and shares no code with it; the two meet only through the seeded input
generator, which holds none of the method's arithmetic.

The arithmetic lives in ``ramnet_oracle.c`` (plain C, double precision, one
straight-line loop per step of the RAM-Net project page's description).  This module
compiles it with gcc on first use and wraps it with ctypes over numpy arrays.
Every array argument is converted to a C-contiguous float64 / int32 / uint8 copy, so
bf16 or fp32 inputs reach the oracle as their exact values.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ramnet_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libramnet_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libramnet_oracle.so`` (no fast-math, no FMA
    contraction) and return its path."""
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c99", "-D_GNU_SOURCE", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-pthread", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Cfg(ctypes.Structure):
    _fields_ = [("d_p", ctypes.c_int32), ("U", ctypes.c_int32), ("K", ctypes.c_int32),
                ("d_v", ctypes.c_int32), ("eps_gsu", ctypes.c_double),
                ("eps_norm", ctypes.c_double), ("renorm", ctypes.c_int32)]


@dataclass(frozen=True)
class OracleConfig:
    """Layer hyper-parameters: M = d_p**U slots, Top-K, value width d_v, the two
    epsilons (readings R8 and R11) and the weight renormalisation switch (R5)."""
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


_P = ctypes.c_void_p


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.ro_digit_score.restype = ctypes.c_int64
            lib.ro_digit_score.argtypes = [ctypes.c_double]
            for name in ("ro_topk_bruteforce", "ro_topk_tree"):
                f = getattr(lib, name)
                f.restype = ctypes.c_int
                f.argtypes = [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P]
            lib.ro_weights.restype = None
            lib.ro_weights.argtypes = [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, ctypes.c_int, _P]
            lib.ro_cape.restype = ctypes.c_int64
            lib.ro_cape.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
            lib.ro_alpha.restype = ctypes.c_double
            lib.ro_alpha.argtypes = [ctypes.c_double, ctypes.c_double]
            lib.ro_decode_addresses.restype = ctypes.c_int
            lib.ro_decode_addresses.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, _P, _P, _P, _P, _P]
            lib.ro_scan_forward.restype = ctypes.c_int
            lib.ro_scan_forward.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int] + [_P] * 13 + [ctypes.c_int]
            lib.ro_decode_step.restype = ctypes.c_int
            lib.ro_decode_step.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int, ctypes.c_int] + \
                [_P] * 11 + [ctypes.c_int, ctypes.c_int]
            _lib = lib
    return _lib


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor: exact widening of bf16/fp32 values
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a):
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def _u8(a):
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.uint8)


def _ptr(a):
    return None if a is None else a.ctypes.data


# ---------------------------------------------------------------- single-token pieces

def digit_score(x: float) -> int:
    """Reading R3: the fixed-point ranking score of one digit logit."""
    return int(_load().ro_digit_score(float(x)))


def topk_bruteforce(x, d_p: int, U: int, K: int):
    """Exact Top-K of one token's logits by scoring all M slots; returns (idx, key)."""
    x = _f64(x).reshape(-1)
    assert x.size == d_p * U
    idx = np.zeros(K, np.int32)
    key = np.zeros(K, np.int64)
    rc = _load().ro_topk_bruteforce(_ptr(x), d_p, U, K, _ptr(idx), _ptr(key))
    if rc != 0:
        raise ValueError(f"ro_topk_bruteforce failed ({rc})")
    return idx, key


def topk_tree(x, d_p: int, U: int, K: int):
    """Exact Top-K by the level-by-level prefix-tree search; returns (idx, key)."""
    x = _f64(x).reshape(-1)
    assert x.size == d_p * U
    idx = np.zeros(K, np.int32)
    key = np.zeros(K, np.int64)
    rc = _load().ro_topk_tree(_ptr(x), d_p, U, K, _ptr(idx), _ptr(key))
    if rc != 0:
        raise ValueError(f"ro_topk_tree failed ({rc})")
    return idx, key


def weights(x, d_p: int, U: int, idx, renorm: int = 1):
    """Product-softmax weights of the given slots (renormalised over them if renorm)."""
    x = _f64(x).reshape(-1)
    idx = _i32(idx).reshape(-1)
    w = np.zeros(idx.size, np.float64)
    _load().ro_weights(_ptr(x), d_p, U, idx.size, _ptr(idx), int(renorm), _ptr(w))
    return w


def cape(idx: int, pos: int, M: int) -> int:
    """Reading R6: cyclic +pos shift of a slot index."""
    return int(_load().ro_cape(int(idx), int(pos), int(M)))


def alpha(w: float, g: float) -> float:
    """Reading R7: GSU retention (1 - w) ** (g / (1 - g)) with its edge rules."""
    return float(_load().ro_alpha(float(w), float(g)))


# ---------------------------------------------------------------- whole-layer calls

def decode_addresses(cfg: OracleConfig, logits, pos0=None, cape_mask=None):
    """logits [B,T,H,U*d_p] -> (idx int32 [B,T,H,K] in rank order, w float64 [B,T,H,K])."""
    x = _f64(logits)
    B, T, H, L = x.shape
    assert L == cfg.L
    pos0, cape_mask = _i32(pos0), _u8(cape_mask)
    idx = np.zeros((B, T, H, cfg.K), np.int32)
    w = np.zeros((B, T, H, cfg.K), np.float64)
    c = cfg._c()
    _load().ro_decode_addresses(ctypes.byref(c), B, T, H, _ptr(x), _ptr(pos0), _ptr(cape_mask),
                                _ptr(idx), _ptr(w))
    return idx, w


def scan_forward(cfg: OracleConfig, k_logits, q_logits, v, g, z, norm_w=None, cape_mask=None,
                 pos0=None, S_in=None, m_in=None, nthreads: int = 0):
    """Prefill scan over [B,T,H,...] inputs; returns (y [B,T,H,d_v], S [B,H,M,d_v], m [B,H,M])
    in float64.  nthreads <= 0 uses every online core (parallel over (b,h) only)."""
    k, q, v, g, z = _f64(k_logits), _f64(q_logits), _f64(v), _f64(g), _f64(z)
    B, T, H, L = k.shape
    assert L == cfg.L and q.shape == k.shape
    assert v.shape == (B, T, H, cfg.d_v) and z.shape == v.shape and g.shape == (B, T, H)
    norm_w, S_in, m_in = _f64(norm_w), _f64(S_in), _f64(m_in)
    cape_mask, pos0 = _u8(cape_mask), _i32(pos0)
    M = cfg.M
    if S_in is not None:
        assert S_in.shape == (B, H, M, cfg.d_v)
    if m_in is not None:
        assert m_in.shape == (B, H, M)
    y = np.zeros((B, T, H, cfg.d_v), np.float64)
    S = np.zeros((B, H, M, cfg.d_v), np.float64)
    m = np.zeros((B, H, M), np.float64)
    c = cfg._c()
    _load().ro_scan_forward(ctypes.byref(c), B, T, H, _ptr(k), _ptr(q), _ptr(v), _ptr(g), _ptr(z),
                            _ptr(norm_w), _ptr(cape_mask), _ptr(pos0), _ptr(S_in), _ptr(m_in),
                            _ptr(y), _ptr(S), _ptr(m), int(nthreads))
    return y, S, m


def decode_step(cfg: OracleConfig, k_logits, q_logits, v, g, z, S, m, pos=None, norm_w=None,
                cape_mask=None, units=None):
    """One decode token per (b,h): k,q [B,H,L], v,z [B,H,d_v], g [B,H], pos [B].
    S [B,H,M,d_v] and m [B,H,M] are float64 numpy arrays updated IN PLACE.
    units = (begin, end) restricts the step to flattened (b*H + h) units in [begin, end).
    Returns y [B,H,d_v] (zeros outside the unit range)."""
    k, q, v, g, z = _f64(k_logits), _f64(q_logits), _f64(v), _f64(g), _f64(z)
    B, H, L = k.shape
    assert L == cfg.L and v.shape == (B, H, cfg.d_v) and g.shape == (B, H)
    assert isinstance(S, np.ndarray) and S.dtype == np.float64 and S.flags.c_contiguous
    assert isinstance(m, np.ndarray) and m.dtype == np.float64 and m.flags.c_contiguous
    assert S.shape == (B, H, cfg.M, cfg.d_v) and m.shape == (B, H, cfg.M)
    norm_w, cape_mask, pos = _f64(norm_w), _u8(cape_mask), _i32(pos)
    y = np.zeros((B, H, cfg.d_v), np.float64)
    ub, ue = (0, B * H) if units is None else units
    c = cfg._c()
    _load().ro_decode_step(ctypes.byref(c), B, H, _ptr(k), _ptr(q), _ptr(v), _ptr(g), _ptr(z),
                           _ptr(norm_w), _ptr(cape_mask), _ptr(pos), _ptr(S), _ptr(m), _ptr(y),
                           int(ub), int(ue))
    return y
