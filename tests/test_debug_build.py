"""The debug build (libnmoe_debug.so, -DNMOE_DEBUG): the same kernels with index and span
checks that report a failed check through the error word (NMOE_ERR_DEVICE_CHECK) and
skip the access it guards. It must export the same entry points, give the release
build's outputs bit for bit on valid inputs with a clean error word, and report, rather
than follow, a token-list span that runs backwards."""

import ctypes as C
import os
import subprocess
import sys
from pathlib import Path

import pytest

import diffusion_transformer_moe_b200 as nm
from diffusion_transformer_moe_b200 import _lib as L

ROOT = Path(__file__).resolve().parents[1]
DEBUG_LIB = ROOT / "diffusion_transformer_moe_b200" / "libnmoe_debug.so"


def test_debug_library_exports_every_entry_point_and_says_so():
    lib = C.CDLL(str(DEBUG_LIB))
    for name in L.EXPORTS:
        assert hasattr(lib, name), name
    lib.nmoe_build_info.restype = C.c_char_p
    assert b"debug checks" in lib.nmoe_build_info()
    assert b"debug checks" not in nm.lib().nmoe_build_info()


_RUN = """
import sys, torch
sys.path.insert(0, sys.argv[1])
import diffusion_transformer_moe_b200 as nm
from diffusion_transformer_moe_b200 import ep, inputs as I
assert ("debug checks" in nm.build_info()) == (sys.argv[3] == "1")
outs = {}
w = I.WORKLOADS["1024px_cfg"]
a = {k: v.cuda() for k, v in I.make_inputs(w).items()}
outs["1024px"] = nm.forward(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], w.C)
b = {k: v.cuda() for k, v in I.make_small(300, 136, 5, 200, "bf16", seed=77).items()}
g = torch.Generator().manual_seed(3)
sh = tuple((torch.randn(*s, generator=g) / s[0] ** 0.5).to(torch.bfloat16).cuda()
           for s in ((136, 104), (136, 104), (104, 136)))
outs["block"] = nm.forward(b["x"], b["W_r"], b["W1"], b["W3"], b["W2"], 20, n_segments=3,
                           shared=sh, residual=b["x"],
                           gate2=torch.randn(3, 136, generator=g).cuda())
outs["gather4"] = nm.forward(b["x"], b["W_r"], b["W1"], b["W3"], b["W2"], 37,
                             tma_gather=True)
st, buf, sc, rc = ep.prepare(b["x"], b["W_r"], b["W1"][:3].contiguous(),
                             b["W3"][:3].contiguous(), b["W2"][:3].contiguous(), 37, 5, 2, 0)
outs["ep_send"] = buf
torch.cuda.synchronize()
assert nm.get_last_error() == 0
torch.save({k: v.cpu() for k, v in outs.items()}, sys.argv[2])
"""


def _run(tmp_path, debug):
    out = tmp_path / ("debug.pt" if debug else "release.pt")
    env = dict(os.environ, NMOE_DEBUG="1" if debug else "0")
    r = subprocess.run([sys.executable, "-c", _RUN, str(ROOT), str(out), "1" if debug else "0"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    import torch
    return torch.load(out)


@pytest.mark.gpu
def test_debug_build_gives_the_release_outputs_with_a_clean_error_word(tmp_path):
    import torch
    rel, dbg = _run(tmp_path, False), _run(tmp_path, True)
    assert rel.keys() == dbg.keys()
    for k in rel:
        assert torch.equal(rel[k], dbg[k]), k


_BACKWARDS = """
import sys, torch
sys.path.insert(0, sys.argv[1])
import diffusion_transformer_moe_b200 as nm
from diffusion_transformer_moe_b200 import _lib as L
assert "debug checks" in nm.build_info()
# 8 tokens over 16 rows of Y; token 3's span runs backwards (rows 9 .. 6). Every value
# lies inside Y, so even the unchecked kernel would stay in bounds.
Y = torch.randn(16, 64, device="cuda")
tok_ptr = torch.tensor([0, 2, 4, 9, 6, 10, 12, 14, 16], dtype=torch.int32, device="cuda")
out = torch.empty(8, 64, device="cuda")
st = L.lib().nmoe_combine_tokens(Y.data_ptr(), tok_ptr.data_ptr(), 8, 64, 0, 8, L.NMOE_F32,
                                 L.NMOE_F32, out.data_ptr(), L._stream())
assert st == 0, st
assert nm.get_last_error() == 6   # NMOE_ERR_DEVICE_CHECK
good = torch.tensor([0, 2, 4, 6, 9, 10, 12, 14, 16], dtype=torch.int32, device="cuda")
st = L.lib().nmoe_combine_tokens(Y.data_ptr(), good.data_ptr(), 8, 64, 0, 8, L.NMOE_F32,
                                 L.NMOE_F32, out.data_ptr(), L._stream())
assert st == 0 and nm.get_last_error() == 0
ref = torch.stack([Y[int(good[t]):int(good[t + 1])].sum(0) for t in range(8)])
assert torch.allclose(out, ref, atol=1e-5)
"""


@pytest.mark.gpu
def test_debug_build_reports_a_backwards_token_span():
    env = dict(os.environ, NMOE_DEBUG="1")
    r = subprocess.run([sys.executable, "-c", _BACKWARDS, str(ROOT)], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-3000:]
