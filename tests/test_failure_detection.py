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
