"""Concurrent first calls from two host threads.

The chunked kernel's launch set-up (its shared-memory attribute and the SM
count that picks the launch shape) is done once per device under a lock. A
fresh process is needed so that the two threads' calls really are the first
ones: each thread runs a chunked prefill on its own stream and inputs, and
both results must equal the same calls made one after the other.
"""
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

SCRIPT = r"""
import sys, threading
sys.path.insert(0, %(root)r)
import torch
from gated_delta_rule_61_b200 import kda
from gated_delta_rule_61_b200.inputs import prefill_inputs

dev = torch.device("cuda")
cases = [prefill_inputs(2, 200, 3, 128, 128, dtype=torch.bfloat16, seed=s, init_std=0.1,
                        device=dev) for s in (1, 2)]
streams = [torch.cuda.Stream() for _ in cases]
outs = [None, None]
errors = []
start = threading.Barrier(2)

def run(i):
    try:
        start.wait()
        g = cases[i]
        with torch.cuda.stream(streams[i]):
            outs[i] = kda.prefill(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"],
                                  init_state=g["init_state"], chunk=64, stream=streams[i])
        streams[i].synchronize()
    except Exception as e:   # reported by the parent
        errors.append(repr(e))

threads = [threading.Thread(target=run, args=(i,)) for i in range(2)]
for t in threads:
    t.start()
for t in threads:
    t.join()
assert not errors, errors
for i, g in enumerate(cases):
    o, s = kda.prefill(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"],
                       init_state=g["init_state"], chunk=64)
    torch.cuda.synchronize()
    assert torch.equal(o, outs[i][0]) and torch.equal(s, outs[i][1]), i
st, detail = kda.device_status()
assert st == kda.KDA_OK, (st, detail)
print("threads ok")
"""


def test_first_calls_from_two_threads():
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", SCRIPT % {"root": root}], capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "threads ok" in r.stdout
