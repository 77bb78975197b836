"""nmoe_forward_noalloc: the layer for callers that cannot allocate device memory.

It keeps all of its scratch in one fixed 128 MiB device array instead of allocating,
so it must give the same outputs as nmoe_forward, call after call, even though every
call reuses (and leaves behind) the previous call's scratch contents. This file is
collected last so that a run that stops at the first failure has run everything else.
"""

import ctypes as C

import numpy as np
import pytest
import torch

import diffusion_transformer_moe_b200 as nm
from diffusion_transformer_moe_b200 import inputs as I

pytestmark = pytest.mark.gpu

BF16_REL, BF16_ABS = 1e-2, 5e-2


def _noalloc(x, W_r, W1, W3, W2, C_, out):
    T, d = x.shape
    E, _, F = W1.shape
    return nm.lib().nmoe_forward_noalloc(
        x.data_ptr(), W_r.data_ptr(), W1.data_ptr(), W3.data_ptr(), W2.data_ptr(), T, d, E,
        F, C_, out.data_ptr(), C.c_void_p(torch.cuda.current_stream().cuda_stream))


def _close(y, ref):
    y = y.float().cpu().numpy().astype(np.float64)
    r = ref.float().cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(y - r) / max(np.linalg.norm(r), 1e-300)
    assert rel <= BF16_REL, rel
    assert np.abs(y - r).max() <= BF16_ABS


def test_noalloc_matches_forward_on_two_calls_in_a_row():
    shape = dict(T=1024, d=256, E=8, F=256)
    C_ = 128
    for seed in (3, 4):  # two calls, different inputs: the second sees the first's scratch
        a = I.make_small(shape["T"], shape["d"], shape["E"], shape["F"], "bf16", seed=seed)
        dev = {k: v.cuda() for k, v in a.items()}
        ref = nm.forward(dev["x"], dev["W_r"], dev["W1"], dev["W3"], dev["W2"], C_)
        out = torch.full_like(dev["x"], float("nan"))
        st = _noalloc(dev["x"], dev["W_r"], dev["W1"], dev["W3"], dev["W2"], C_, out)
        assert st == 0, nm.lib().nmoe_status_str(st)
        torch.cuda.synchronize()
        assert nm.get_last_error() == 0
        _close(out, ref)


def test_noalloc_matches_forward_on_the_1024px_workload():
    w = I.WORKLOADS["1024px_cfg"]
    a = I.make_inputs(w)
    dev = {k: v.cuda() for k, v in a.items()}
    ref = nm.forward(dev["x"], dev["W_r"], dev["W1"], dev["W3"], dev["W2"], w.C)
    for _ in range(2):  # the second call sees the first call's scratch
        out = torch.full_like(dev["x"], float("nan"))
        st = _noalloc(dev["x"], dev["W_r"], dev["W1"], dev["W3"], dev["W2"], w.C, out)
        assert st == 0, nm.lib().nmoe_status_str(st)
        torch.cuda.synchronize()
        assert nm.get_last_error() == 0
        # the same kernels on the same inputs: the same bits
        assert torch.equal(out, ref)


def test_noalloc_rejects_sizes_beyond_its_capacity():
    # the batch-4 workload needs far more than 128 MiB of scratch: rejected, nothing runs
    w = I.WORKLOADS["batch4_1024px_cfg"]
    need = nm.workspace_size(w.T, w.d, w.E, w.F, w.C)
    assert need > (128 << 20)
    buf = torch.empty(64, dtype=torch.bfloat16, device="cuda")
    p = buf.data_ptr()
    st = nm.lib().nmoe_forward_noalloc(p, p, p, p, p, w.T, w.d, w.E, w.F, w.C, p + 64,
                                       C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 3  # NMOE_ERR_WORKSPACE
