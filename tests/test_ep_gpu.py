"""Expert parallelism on one GPU: the ranks' halves (``ep.prepare`` / ``ep.finish``) run
one after another in one process, and the all-to-all between them is done by handing
each rank the slices of the others' send buffers; every rank's output rows must equal
the single-GPU layer's, bit for bit."""

import pytest
import torch

import diffusion_transformer_moe_b200 as nm
from diffusion_transformer_moe_b200 import ep
from diffusion_transformer_moe_b200 import inputs as I

pytestmark = pytest.mark.gpu


def _emulated_ep(dev, C_, E, world, n_segments=1):
    states, sends = [], []
    for r in range(world):
        lo, hi = ep.split_range(E, world, r)
        st, buf, send_counts, recv_counts = ep.prepare(
            dev["x"], dev["W_r"], dev["W1"][lo:hi].contiguous(), dev["W3"][lo:hi].contiguous(),
            dev["W2"][lo:hi].contiguous(), C_, E, world, r, n_segments=n_segments)
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


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("dtype,T,d,E,F,C_,nseg", [
    ("bf16", 1024, 256, 8, 256, 128, 1),     # tensor-core path
    ("bf16", 768, 136, 6, 200, 100, 2),      # ragged sizes, selection per segment
    ("f32", 256, 128, 6, 96, 40, 1),         # CUDA-core path
])
def test_expert_parallel_equals_one_gpu(world, dtype, T, d, E, F, C_, nseg):
    a = I.make_small(T, d, E, F, dtype, seed=T + E)
    dev = {k: v.cuda() for k, v in a.items()}
    ref = nm.forward(dev["x"], dev["W_r"], dev["W1"], dev["W3"], dev["W2"], C_,
                     n_segments=nseg)
    out = _emulated_ep(dev, C_, E, world, nseg)
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
        assert torch.equal(out, ref)
    finally:
        dist.destroy_process_group()
