"""Calls from several host threads at once (the C ABI promises thread-safe calls: its only
process-wide state is per-device setup, made once under locks).

The threads start in a fresh process before any other call into the library. Their
first calls therefore race on that one-time setup: kernel attributes, the tensor-map
encoder, the 2-CTA pair count. Each thread then runs the layer on its own stream with
its own workspace. Every thread's output must equal a single-threaded call's, bit for
bit."""

import subprocess
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]

pytestmark = pytest.mark.gpu

_SCRIPT = r"""
import sys, threading
import torch
sys.path.insert(0, sys.argv[1])
import diffusion_transformer_moe_b200 as nm
from diffusion_transformer_moe_b200 import inputs as I

# (T, d, E, F, C): large experts (pair down GEMM, two row blocks per gate/up item), a
# middle shape, and the 1024 px layer's shape (one-CTA GEMMs, ring combine)
cases = [(2048, 256, 4, 192, 1100), (2048, 512, 8, 256, 256), (8192, 2048, 64, 1024, 128)]
data = []
for T, d, E, F, C_ in cases:
    a = {k: v.cuda() for k, v in I.make_small(T, d, E, F, "bf16", seed=T + E).items()}
    data.append((a, C_))
torch.cuda.synchronize()

n_threads = 4
outs = [[None] * len(cases) for _ in range(n_threads)]
errors = []
go = threading.Barrier(n_threads)

def work(t):
    try:
        s = torch.cuda.Stream()
        go.wait()
        for ci, (a, C_) in enumerate(data):
            out = torch.empty_like(a["x"])
            with torch.cuda.stream(s):
                for _ in range(3):
                    nm.forward(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C_, out=out,
                               stream=s)
            s.synchronize()
            outs[t][ci] = out
    except Exception as e:  # reported by the main thread
        errors.append(repr(e))

threads = [threading.Thread(target=work, args=(t,)) for t in range(n_threads)]
for th in threads:
    th.start()
for th in threads:
    th.join()
assert not errors, errors
for ci, (a, C_) in enumerate(data):
    want = nm.forward(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C_)
    torch.cuda.synchronize()
    for t in range(n_threads):
        assert torch.equal(outs[t][ci], want), (t, cases[ci])
assert nm.get_last_error() == 0
print("ok")
"""


def test_threads_racing_on_first_calls_match_one_thread():
    r = subprocess.run([sys.executable, "-c", _SCRIPT, str(ROOT)], capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, (r.stdout[-2000:], r.stderr[-4000:])
    assert r.stdout.strip().endswith("ok")
