"""Expert parallelism on one GPU.

Emulated: the ranks' halves (``ep.prepare`` / ``ep.finish``) run one after another in one
process, and the all-to-all between them is done by handing each rank the slices of the
others' send buffers. Real ranks: separate processes (each its own CUDA context on the
one GPU; no kernel of one waits on another's) exchange rows through a gloo group over
host memory. Every rank's output rows must equal the single-GPU layer's, bit for bit,
and the whole output must match the oracle at the layer's tolerances."""

import os
import socket
import subprocess
import sys
from pathlib import Path

import numpy as np
import pytest
import torch

import diffusion_transformer_moe_b200 as nm
from diffusion_transformer_moe_b200 import ep
from diffusion_transformer_moe_b200 import inputs as I

pytestmark = pytest.mark.gpu


def _emulated_ep(dev, C_, E, world, n_segments=1, exact=False):
    states, sends = [], []
    for r in range(world):
        lo, hi = ep.split_range(E, world, r)
        st, buf, send_counts, recv_counts = ep.prepare(
            dev["x"], dev["W_r"], dev["W1"][lo:hi].contiguous(), dev["W3"][lo:hi].contiguous(),
            dev["W2"][lo:hi].contiguous(), C_, E, world, r, n_segments=n_segments,
            exact=exact)
        states.append((st, recv_counts))
        sends.append((buf, send_counts))
    outs = []
    for r, (st, recv_counts) in enumerate(states):
        parts = []
        for g in range(world):  # rows g sends to r: g's buffer after the parts for ranks < r
            buf, counts = sends[g]
            at = sum(counts[:r])
            parts.append(buf[at:at + counts[r]])
            assert counts[r] == recv_counts[g]
        outs.append(ep.finish(st, torch.cat(parts)))
    torch.cuda.synchronize()
    assert nm.get_last_error() == 0
    return torch.cat(outs)


@pytest.mark.parametrize("exact", [False, True])
@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("dtype,T,d,E,F,C_,nseg", [
    ("bf16", 1024, 256, 8, 256, 128, 1),     # tensor-core path
    ("bf16", 768, 136, 6, 200, 100, 2),      # ragged sizes, selection per segment
    ("f32", 256, 128, 6, 96, 40, 1),         # CUDA-core path
    ("bf16", 2048, 256, 8, 192, 384, 1),     # the pair down GEMM on each rank's experts
    ("bf16", 2048, 256, 4, 192, 1100, 1),    # and two row blocks per gate/up item
])
def test_expert_parallel_equals_one_gpu(world, dtype, T, d, E, F, C_, nseg, exact):
    a = I.make_small(T, d, E, F, dtype, seed=T + E)
    dev = {k: v.cuda() for k, v in a.items()}
    ref = nm.forward(dev["x"], dev["W_r"], dev["W1"], dev["W3"], dev["W2"], C_,
                     n_segments=nseg)
    out = _emulated_ep(dev, C_, E, world, nseg, exact)
    assert torch.equal(out, ref)


def test_expert_parallel_1024px_equals_one_gpu():
    w = I.WORKLOADS["1024px_cfg"]
    a = I.make_inputs(w)
    dev = {k: v.cuda() for k, v in a.items()}
    ref = nm.forward(dev["x"], dev["W_r"], dev["W1"], dev["W3"], dev["W2"], w.C)
    out = _emulated_ep(dev, w.C, w.E, 4)
    assert torch.equal(out, ref)


def test_forward_over_a_one_rank_nccl_group():
    # the torch.distributed path itself (the all-to-all with one rank moves nothing)
    import socket
    import torch.distributed as dist
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", world_size=1,
                            rank=0, device_id=torch.device("cuda", 0))
    try:
        a = I.make_small(512, 128, 4, 128, "bf16", seed=9)
        dev = {k: v.cuda() for k, v in a.items()}
        ref = nm.forward(dev["x"], dev["W_r"], dev["W1"], dev["W3"], dev["W2"], 64)
        out = ep.forward(dev["x"], dev["W_r"], dev["W1"], dev["W3"], dev["W2"], 64, 4)
        torch.cuda.synchronize()
        assert nm.get_last_error() == 0
        assert torch.equal(out, ref)
    finally:
        dist.destroy_process_group()


# -- real ranks: one process each, rows exchanged through gloo ------------------------------

_EP_RANK = """
import datetime, os, sys, torch
sys.path.insert(0, sys.argv[1])
import torch.distributed as dist
import diffusion_transformer_moe_b200 as nm
from diffusion_transformer_moe_b200 import ep, inputs as I
spec, exact, outdir = sys.argv[2], sys.argv[3] == "1", sys.argv[4]
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
torch.cuda.set_device(0)
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=300))
if spec in I.WORKLOADS:
    w = I.WORKLOADS[spec]
    a, C_, E, nseg = I.make_inputs(w), w.C, w.E, w.segments
else:
    T, d, E, F, C_, nseg = map(int, spec.split(","))
    a = I.make_small(T, d, E, F, "bf16", seed=T + E)
lo, hi = ep.split_range(E, world, rank)
dev = {k: v.cuda() for k, v in a.items()}
out = ep.forward(dev["x"], dev["W_r"], dev["W1"][lo:hi].contiguous(),
                 dev["W3"][lo:hi].contiguous(), dev["W2"][lo:hi].contiguous(), C_, E,
                 n_segments=nseg, exact=exact)
torch.cuda.synchronize()
assert nm.get_last_error() == 0
torch.save(out.cpu(), os.path.join(outdir, f"rank{rank}.pt"))
dist.barrier()
dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def _run_ranks(spec, world, exact, tmp):
    root = str(Path(__file__).resolve().parents[1])
    port = _free_port()
    procs = []
    for rank in range(world):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK="0",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", _EP_RANK, root, spec,
                                       "1" if exact else "0", str(tmp)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                      text=True))
    errs = []
    for p in procs:
        try:
            _, e = p.communicate(timeout=900)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            pytest.fail("an expert-parallel rank did not finish")
        errs.append((p.returncode, e[-3000:]))
    for rc, e in errs:
        assert rc == 0, e
    return torch.cat([torch.load(tmp / f"rank{r}.pt") for r in range(world)])


@pytest.mark.parametrize("spec,world,exact", [
    ("1024px_cfg", 2, False),             # the 1024 px layer, half the experts per rank
    ("768,136,6,200,100,2", 3, True),     # ragged sizes, per-segment selection, exact counts
])
def test_expert_parallel_ranks_match_the_oracle(spec, world, exact, tmp_path):
    from oracle import nmoe_oracle as O
    from tests.test_parity_gpu import _check_out
    out = _run_ranks(spec, world, exact, tmp_path)
    if spec in I.WORKLOADS:
        w = I.WORKLOADS[spec]
        a, C_, nseg = I.make_inputs(w), w.C, w.segments
    else:
        T, d, E, F, C_, nseg = map(int, spec.split(","))
        a = I.make_small(T, d, E, F, "bf16", seed=T + E)
    dev = {k: v.cuda() for k, v in a.items()}
    E = a["W_r"].shape[1]
    idx = torch.empty(E, nseg * C_, dtype=torch.int32, device="cuda")
    ref = nm.forward(dev["x"], dev["W_r"], dev["W1"], dev["W3"], dev["W2"], C_,
                     n_segments=nseg, idx_out=idx)
    torch.cuda.synchronize()
    assert torch.equal(out, ref.cpu())
    sel = idx.cpu().numpy()
    del dev
    r = O.layer(I.to_numpy_f64(a["x"]), I.to_numpy_f64(a["W_r"]), a["W1"].float().numpy(),
                a["W3"].float().numpy(), a["W2"].float().numpy(), C_, selection=sel,
                n_segments=nseg)
    _check_out(out, r["out"], "bf16")
