"""The range-checking build (libramnet_debug.so, compiled with RAMNET_DEBUG) on the small
parity cases.

In that build every kernel checks the slot indices, ring positions and event fields it
computes before using them and records a failed check in the device status word; the
parity tests call ramnet_sync_status after each kernel, so any failed check fails them.
Runs the small cases of test_gpu_parity.py in a child process with RAMNET_DEBUG=1.
"""
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

SMALL_CASES = ("tiny or test_scan_matches_oracle or test_route_events_match_oracle or "
               "test_decode_step_matches_oracle_over_steps or test_decode_addresses_matches_oracle or "
               "write_gate_edges or every_slot_selected")


def test_debug_build_small_parity_cases():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from sparse_slot_recurrent_b200 import build as build_mod
    build_mod.build(debug=True)
    env = dict(os.environ, RAMNET_DEBUG="1", PYTHONPATH=ROOT)
    which = subprocess.run([sys.executable, "-c", "from sparse_slot_recurrent_b200 import ramnet; ramnet.load(); "
                            "print(ramnet.LIB_PATH)"], env=env, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert which.returncode == 0, which.stderr
    assert which.stdout.strip().endswith("libramnet_debug.so")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join("tests", "test_gpu_parity.py"), "-q", "-x",
                        "-m", "gpu", "-k", SMALL_CASES, "-p", "no:cacheprovider"],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
