"""Failure detection: a bounded device wait that runs out is reported, not hung.

The self-test kernel waits, through the same bounded-wait routine the prefill scan uses,
on a barrier that nothing signals.  The wait must give up after its limit and leave
RAMNET_ERR_TIMEOUT in the status word; ramnet_sync_status reports it once and clears it,
and the context stays usable (a scan afterwards still matches the oracle).  Nothing here
faults, traps or hangs the GPU.  Host-side argument checks run on CPU.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from sparse_slot_recurrent_b200 import ramnet
from sparse_slot_recurrent_b200.workloads import WORKLOADS, generate


def test_scan_wait_limit_rejects_bad_limit_on_host():
    lib = ramnet.load()
    assert lib.ramnet_set_scan_wait_limit(2000001) == ramnet.RAMNET_ERR_INVALID_ARG
    assert "limit_us" in ramnet.last_error()
    assert lib.ramnet_set_scan_wait_limit(0) == ramnet.RAMNET_OK


def test_selftest_rejects_bad_limit_on_host():
    lib = ramnet.load()
    assert lib.ramnet_selftest_wait_timeout(0, None) == ramnet.RAMNET_ERR_INVALID_ARG
    assert lib.ramnet_selftest_wait_timeout(2000001, None) == ramnet.RAMNET_ERR_INVALID_ARG
    assert "limit_us" in ramnet.last_error()


@pytest.mark.gpu
def test_wait_timeout_is_reported_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    ramnet.sync_status()  # start from a clear status word
    t0 = time.perf_counter()
    ramnet.selftest_wait_timeout(20000)  # 20 ms
    with pytest.raises(ramnet.RamnetError) as e:
        ramnet.sync_status()
    elapsed = time.perf_counter() - t0
    assert e.value.status == ramnet.RAMNET_ERR_TIMEOUT
    assert 0.015 <= elapsed < 5.0
    ramnet.sync_status()  # cleared: no error the second time
    w = WORKLOADS["tiny"]
    cfg = ramnet.Config(d_p=w.d_p, U=w.U, K=w.K, d_v=w.d_v)
    ocfg = oracle.OracleConfig(d_p=w.d_p, U=w.U, K=w.K, d_v=w.d_v)
    inp = generate(w, seed=0)
    d = {k: v.cuda() for k, v in inp.items() if torch.is_tensor(v)}
    y, S, m = ramnet.scan_forward(cfg, d["k_logits"], d["q_logits"], d["v"], d["g"], d["z"],
                                  cape_mask=d["cape_mask"], pos0=d["pos0"])
    ramnet.sync_status()
    oy, oS, om = oracle.scan_forward(ocfg, inp["k_logits"], inp["q_logits"], inp["v"], inp["g"], inp["z"],
                                     cape_mask=inp["cape_mask"], pos0=inp["pos0"])
    assert float(np.abs(y.cpu().double().numpy() - np.asarray(oy)).max()) <= 1e-5


@pytest.mark.gpu
def test_recurrence_wait_timeout_is_reported_and_context_survives():
    """The prefill recurrence itself with a 1 us limit on its waits: its hand-overs take longer
    (the first staged chunk alone needs a DRAM round trip), so waits run out.  The kernel must
    record RAMNET_ERR_TIMEOUT and end by itself; with the default limit restored, a scan
    afterwards matches the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    w = WORKLOADS["prefill_340m_top8"].with_(B=1, H=2, T=1024)
    cfg = ramnet.Config(d_p=w.d_p, U=w.U, K=w.K, d_v=w.d_v)
    inp = generate(w, seed=3)
    d = {k: v.cuda() for k, v in inp.items() if torch.is_tensor(v)}
    ramnet.sync_status()
    ramnet.set_scan_wait_limit(1)
    try:
        t0 = time.perf_counter()
        ramnet.scan_forward(cfg, d["k_logits"], d["q_logits"], d["v"], d["g"], d["z"], cape_mask=d["cape_mask"],
                            pos0=d["pos0"])
        with pytest.raises(ramnet.RamnetError) as e:
            ramnet.sync_status()
        assert e.value.status == ramnet.RAMNET_ERR_TIMEOUT
        assert time.perf_counter() - t0 < 10.0
    finally:
        ramnet.set_scan_wait_limit(0)
    ramnet.sync_status()
    t = WORKLOADS["tiny"]
    tcfg = ramnet.Config(d_p=t.d_p, U=t.U, K=t.K, d_v=t.d_v)
    ocfg = oracle.OracleConfig(d_p=t.d_p, U=t.U, K=t.K, d_v=t.d_v)
    tin = generate(t, seed=0)
    td = {k: v.cuda() for k, v in tin.items() if torch.is_tensor(v)}
    y, S, m = ramnet.scan_forward(tcfg, td["k_logits"], td["q_logits"], td["v"], td["g"], td["z"],
                                  cape_mask=td["cape_mask"], pos0=td["pos0"])
    ramnet.sync_status()
    oy, oS, om = oracle.scan_forward(ocfg, tin["k_logits"], tin["q_logits"], tin["v"], tin["g"], tin["z"],
                                     cape_mask=tin["cape_mask"], pos0=tin["pos0"])
    assert float(np.abs(y.cpu().double().numpy() - np.asarray(oy)).max()) <= 1e-5
    assert float(np.abs(S.cpu().double().numpy() - np.asarray(oS)).max()) <= 1e-5
