"""The expert-parallel exchange on the CPU: gloo ranks started the way torchrun starts
them run ``ep.all_to_all_rows`` with the static split sizes of ``ep.exchange_plan``, each
rank's buffer for every destination tagged with (sender, destination, row); every rank
must receive exactly its slices, in rank order, padded rows included."""

import json
import os
import socket
import subprocess
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]

_RANK = """
import datetime, json, os, sys
sys.path.insert(0, sys.argv[1])
import torch
import torch.distributed as dist
from diffusion_transformer_moe_b200 import ep
E, Ce, d = int(sys.argv[2]), int(sys.argv[3]), 8
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
send_splits, recv_splits = ep.exchange_plan(E, Ce, world, rank)
rows = []
for dst, n in enumerate(send_splits):
    for i in range(n):
        rows.append([1000.0 * rank + 100.0 * dst + i] * d)
send = torch.tensor(rows, dtype=torch.float32).view(-1, d)
recv = ep.all_to_all_rows(send, send_splits, recv_splits)
dist.barrier()
dist.destroy_process_group()
print(json.dumps({"rank": rank, "recv": recv[:, 0].tolist(), "recv_splits": recv_splits,
                  "row_ok": bool((recv == recv[:, :1]).all())}))
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,E,Ce", [(2, 8, 4), (3, 7, 3)])
def test_padded_exchange_delivers_every_slice_in_rank_order(world, E, Ce):
    port = _free_port()
    procs = []
    for rank in range(world):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", _RANK, str(ROOT), str(E), str(Ce)],
                                      env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            o, e = p.communicate(timeout=180)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            pytest.fail("a gloo rank did not finish")
        assert p.returncode == 0, e[-2000:]
        outs.append(json.loads(o.strip().splitlines()[-1]))
    from diffusion_transformer_moe_b200 import ep
    for r in outs:
        me = r["rank"]
        assert r["row_ok"]
        want = []
        for src in range(world):
            n = ep.exchange_plan(E, Ce, world, src)[0][me]
            assert n == r["recv_splits"][src]
            want += [1000.0 * src + 100.0 * me + i for i in range(n)]
        assert r["recv"] == want
