"""The standalone row gather / scatter (nmoe_rows_gather, nmoe_rows_scatter) on the GPU.

The gather with rows = the chosen tokens idx [E, Ce] is the grouped-matmul path's permute
into contiguous per-expert blocks (NucleusMoE-Image walkthrough, section 6); the layer
fuses it into the gate/up GEMM, and this copy stands alone for expert parallelism and
for its own bandwidth figure. Index work: every result must equal plain indexing of the
same tensors on the host, bit for bit."""

import pytest
import torch

import diffusion_transformer_moe_b200 as nm
from diffusion_transformer_moe_b200 import _lib as L
from diffusion_transformer_moe_b200 import inputs as I

pytestmark = pytest.mark.gpu


def _host_gather(src, rows):
    out = torch.zeros(rows.numel(), src.shape[1], dtype=src.dtype)
    keep = rows >= 0
    out[keep] = src[rows[keep].long()]
    return out


@pytest.mark.parametrize("n_src,row_bytes,n,dtype", [
    (8192, 4096, 8192, torch.bfloat16),    # 1024 px rows of x: one round of 8 loads a lane
    (4096, 8192, 3001, torch.float32),     # fp32 Y rows (EP): two rounds, ragged count
    (500, 48, 777, torch.float32),         # 3 units per row: most lanes idle
    (100, 16, 33, torch.float32),          # a single unit per row
    (300, 4096 + 16, 129, torch.bfloat16), # 257 units: a second round of one unit
])
def test_gather_equals_host_indexing(n_src, row_bytes, n, dtype):
    g = torch.Generator().manual_seed(n_src + n)
    cols = row_bytes // torch.tensor([], dtype=dtype).element_size()
    src = torch.randn(n_src, cols, generator=g).to(dtype)
    rows = torch.randint(0, n_src, (n,), generator=g, dtype=torch.int32)
    rows[torch.randperm(n, generator=g)[: n // 7]] = -1      # padding rows -> zeros
    rows[: min(5, n)] = rows[0]                                # repeated rows
    out = nm.gather_rows(src.cuda(), rows.cuda())
    torch.cuda.synchronize()
    assert torch.equal(out.cpu(), _host_gather(src, rows))


def test_gather_of_the_layers_own_selection_is_each_experts_block():
    w = I.WORKLOADS["1024px_cfg"]
    a = I.make_inputs(w, seed=3)
    x, W_r = a["x"].cuda(), a["W_r"].cuda()
    _, scores_t = nm.router(x, W_r, n_segments=w.segments)
    idx = nm.select(scores_t, w.C, n_segments=w.segments, csr=False)[0]
    packed = nm.gather_rows(x, idx)
    torch.cuda.synchronize()
    assert packed.shape == (w.E * w.Ce, w.d)
    assert torch.equal(packed.cpu(), a["x"][idx.cpu().view(-1).long()])
    assert nm.get_last_error() == 0


def test_scatter_writes_listed_rows_and_skips_padding():
    g = torch.Generator().manual_seed(11)
    n_dst, n, cols = 2000, 1500, 520         # 2080-byte fp32 rows: 130 units
    src = torch.randn(n, cols, generator=g)
    rows = torch.randperm(n_dst, generator=g)[:n].to(torch.int32)
    rows[::9] = -1
    dst0 = torch.randn(n_dst, cols, generator=g)
    dst = dst0.cuda()
    r = rows.cuda()
    L._check(L.lib().nmoe_rows_scatter(src.cuda().data_ptr(), r.data_ptr(), n, cols * 4,
                                       dst.data_ptr(), L._stream(None)), "nmoe_rows_scatter")
    torch.cuda.synchronize()
    want = dst0.clone()
    keep = rows >= 0
    want[rows[keep].long()] = src[keep]
    assert torch.equal(dst.cpu(), want)


def test_empty_gather_is_a_no_op():
    src = torch.ones(4, 8, dtype=torch.float32, device="cuda")
    rows = torch.empty(0, dtype=torch.int32, device="cuda")
    out = nm.gather_rows(src, rows)
    torch.cuda.synchronize()
    assert out.shape == (0, 8)
