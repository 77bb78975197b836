"""The C ABI library loads, exports what include/nmoe.h declares, and rejects bad
arguments on the host before touching CUDA (CPU only: no compute call is made)."""

import ctypes as C
import os
import re

import pytest

import diffusion_transformer_moe_b200 as nm
from diffusion_transformer_moe_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"NMOE_API\s+[\w\s\*]*?\b(nmoe_\w+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    lib = nm.lib()
    declared = _declared()
    assert declared, "no declarations found"
    assert declared == set(L.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name


def test_options_struct_matches_defaults():
    o = L.Options()
    o.wait_budget_ns = 12345  # the last field: init must reach it at the same offset
    nm.lib().nmoe_options_init(C.byref(o))
    assert o.wait_budget_ns == 0
    assert (o.dtype, o.score_fn, o.combine, o.n_segments, o.host_io) == (0, 0, 0, 1, 0)
    assert o.route_scale == 1.0 and not o.workspace and not o.trace
    assert not o.router_x and not o.residual and o.expert_end == 0


def test_status_strings_and_build_info():
    lib = nm.lib()
    for s in range(8):
        assert lib.nmoe_status_str(s)
    assert b"sm_100a" in lib.nmoe_build_info()


FAKE = 1 << 20  # a 16-byte aligned non-null address; never dereferenced (checks fail first)


@pytest.mark.parametrize("args,expect", [
    (dict(T=0), 1), (dict(E=0), 1), (dict(E=257), 1), (dict(C=0), 1), (dict(C=65), 1),
    (dict(d=12), 2), (dict(F=20), 2), (dict(x=0), 1), (dict(x=FAKE + 8), 1),
    (dict(out=FAKE), 1), (dict(T=(1 << 19) + 64, C=8), 2),
])
def test_forward_rejects_bad_arguments_on_host(args, expect):
    a = dict(x=FAKE, W_r=FAKE + 4096, W1=FAKE + 8192, W3=FAKE + 12288, W2=FAKE + 16384,
             T=64, d=16, E=4, F=16, C=8, out=FAKE + 32768)
    a.update(args)
    st = nm.lib().nmoe_forward(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], a["T"], a["d"],
                               a["E"], a["F"], a["C"], a["out"], None)
    assert st == expect


def test_select_and_router_reject_bad_arguments_on_host():
    lib = nm.lib()
    # C larger than a segment
    assert lib.nmoe_select(FAKE, 64, 4, 33, 2, FAKE, FAKE, None, None, None) == 1
    # T not divisible by the segments
    assert lib.nmoe_select(FAKE, 63, 4, 3, 2, FAKE, FAKE, None, None, None) == 1
    # only one of tok_ptr / tok_ent
    assert lib.nmoe_select(FAKE, 64, 4, 3, 1, FAKE, FAKE, FAKE, None, None) == 1
    # misaligned idx
    assert lib.nmoe_select(FAKE, 64, 4, 3, 1, FAKE + 4, FAKE, None, None, None) == 1
    # no output at all
    assert lib.nmoe_router(FAKE, FAKE, 64, 16, 4, 0, 0, None, 1, None, None, None) == 1
    # bad score function
    assert lib.nmoe_router(FAKE, FAKE, 64, 16, 4, 0, 7, None, 1, FAKE, None, None) == 1


def test_workspace_size_accounts_for_every_buffer():
    T, d, E, F, C_ = 8192, 2048, 64, 1024, 128
    n = nm.workspace_size(T, d, E, F, C_)
    Ce = E * C_
    # default (split) intermediates: H as a bf16 hi/lo pair, Y in fp32 -> 4 bytes each
    blocks = (T + 31) // 32 + 1  # per-expert boundary table of the CSR build
    minimum = (4 * T * E * 2 + 4 * Ce * 4 + 4 * blocks * E + 4 * (T + 1) + 4 * Ce * F
               + 4 * Ce * d)
    assert minimum <= n <= minimum + 16 * 256
    small = nm.workspace_size(T, d, E, F, C_, intermediate="bf16")
    assert small == n - 2 * Ce * F - 2 * Ce * d
    assert nm.workspace_size(T, d, E, F, T + 1) == 0  # invalid sizes give 0
    host = nm.workspace_size(T, d, E, F, C_, host_io=True)
    assert host >= n + 2 * 2 * T * d
    host32 = nm.workspace_size(T, d, E, F, C_, host_io=True, out_f32=True)
    assert host32 >= n + 2 * T * d + 4 * T * d


def test_workspace_holds_a_host_router_input():
    T, d, E, F, C_ = 2048, 1024, 16, 2048, 256
    host = nm.workspace_size(T, d, E, F, C_, host_io=True)
    # a separate router input in host memory is copied into one more [T, d] buffer; on
    # the device it needs none
    o = L.options(host_io=True)
    o.router_x = FAKE
    with_rx = int(nm.lib().nmoe_workspace_size(T, d, E, F, C_, C.byref(o)))
    assert 2 * T * d <= with_rx - host <= 2 * T * d + 256
    o = L.options()
    o.router_x = FAKE
    assert int(nm.lib().nmoe_workspace_size(T, d, E, F, C_, C.byref(o))) == \
        nm.workspace_size(T, d, E, F, C_)


def test_workspace_grows_by_the_shared_expert():
    T, d, E, F, C_, Fs = 8192, 2048, 64, 1024, 128, 1024
    n = nm.workspace_size(T, d, E, F, C_)
    m = nm.workspace_size(T, d, E, F, C_, shared_f=Fs)
    # H hi + lo of the shared expert, one more fp32 Y row and list entry per token
    extra = 4 * T * Fs + 4 * T * d + 4 * T
    assert extra <= m - n <= extra + 3 * 256


def _forward_ex_status(**kw):
    a = dict(x=FAKE, W_r=FAKE + 4096, W1=FAKE + 8192, W3=FAKE + 12288, W2=FAKE + 16384,
             out=FAKE + 32768)
    o = L.Options()
    nm.lib().nmoe_options_init(C.byref(o))
    for k, v in kw.items():
        setattr(o, k, v)
    return nm.lib().nmoe_forward_ex(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], 64, 16, 4,
                                    16, 8, a["out"], None, C.byref(o))


@pytest.mark.parametrize("kw,expect", [
    (dict(shared_w1=FAKE + 65536, shared_f=16), 1),                     # one of three
    (dict(shared_w1=FAKE + 65536, shared_w3=FAKE + 69632, shared_w2=FAKE + 73728,
          shared_f=12), 2),                                              # width % 8
    (dict(shared_w1=FAKE + 65536, shared_w3=FAKE + 69632, shared_w2=FAKE + 73728,
          shared_f=0), 1),
    (dict(gate2=FAKE + 65536), 1),                                       # gate without residual
    (dict(residual=FAKE + 65544), 1),                                    # misaligned
    (dict(residual=FAKE + 32768), 1),                                    # residual is out
    (dict(router_x=FAKE + 65544), 1),                                    # misaligned
    (dict(router_x=FAKE + 32768), 1),                                    # router input is out
])
def test_block_options_are_checked_on_host(kw, expect):
    assert _forward_ex_status(**kw) == expect


@pytest.mark.parametrize("kw,expect", [
    (dict(expert_begin=0, expert_end=2), 1),                    # a rank's range must skip the combine
    (dict(skip_combine=1), 1),                                  # ... and needs a caller workspace
    (dict(expert_begin=0, expert_end=2, skip_combine=1, workspace=FAKE + 65536,
          residual=FAKE + 131072), 1),                          # no residual with expert ranges
])
def test_expert_parallel_options_are_checked_on_host(kw, expect):
    assert _forward_ex_status(**kw) == expect


def test_expert_parallel_calls_check_arguments_on_host():
    lib = nm.lib()
    # t_end beyond T, an empty expert table, a negative capacity, a capacity without a
    # row buffer, misaligned rows, rows not a multiple of 16 B
    assert lib.nmoe_ep_rows(FAKE, FAKE, 64, 4, 8, 0, 65, 0, 2, FAKE, 16, FAKE, None) == 1
    assert lib.nmoe_ep_rows(FAKE, FAKE, 64, 0, 8, 0, 64, 0, 0, FAKE, 16, FAKE, None) == 1
    assert lib.nmoe_ep_rows(FAKE, FAKE, 64, 4, 8, 0, 64, 0, 2, FAKE, -1, FAKE, None) == 1
    assert lib.nmoe_ep_rows(FAKE, FAKE, 64, 4, 8, 0, 64, 0, 2, None, 16, FAKE, None) == 1
    assert lib.nmoe_rows_gather(FAKE + 4, FAKE, 4, 64, FAKE, None) == 1
    assert lib.nmoe_rows_scatter(FAKE, FAKE, 4, 24, FAKE, None) == 1
    assert lib.nmoe_combine_tokens(FAKE, FAKE, 64, 12, 0, 64, 1, 0, FAKE, None) == 2


def test_exchange_plan_is_static_and_symmetric():
    # what rank a sends rank b is what b expects from a; nobody sends itself anything;
    # every buffer holds the sender's whole entry count (an upper bound on any list)
    from diffusion_transformer_moe_b200 import ep
    for E, Ce, world in ((64, 128, 2), (6, 100, 4), (7, 5, 3), (8, 16, 1)):
        plans = [ep.exchange_plan(E, Ce, world, r) for r in range(world)]
        for a in range(world):
            lo, hi = ep.split_range(E, world, a)
            assert plans[a][0][a] == 0 and plans[a][1][a] == 0
            for b in range(world):
                assert plans[a][0][b] == plans[b][1][a]
                if a != b:
                    assert plans[a][0][b] == (hi - lo) * Ce


def test_split_range_covers_every_item_once():
    from diffusion_transformer_moe_b200 import ep
    for n, parts in ((64, 3), (7, 7), (128, 8), (10, 4)):
        got = [ep.split_range(n, parts, i) for i in range(parts)]
        assert got[0][0] == 0 and got[-1][1] == n
        assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
        assert max(e - b for b, e in got) - min(e - b for b, e in got) <= 1


def test_missing_gpu_is_reported_not_crashed():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    # valid arguments on a machine without a device: NMOE_ERR_NO_DEVICE
    st = nm.lib().nmoe_forward(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 16, 4, 16, 8, FAKE + 64, None)
    assert st == 7


def test_the_1024px_workload_fits_the_allocation_free_scratch():
    # nmoe_forward_noalloc promises to run the 1024 px CFG layer in its fixed 128 MiB
    # array: its scratch with default options must stay within that
    from diffusion_transformer_moe_b200 import inputs as I
    w = I.WORKLOADS["1024px_cfg"]
    assert nm.workspace_size(w.T, w.d, w.E, w.F, w.C) <= (128 << 20)
