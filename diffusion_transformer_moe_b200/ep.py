"""Expert parallelism for the layer: one rank per GPU, each holding a contiguous range of
the experts.

Every rank holds all tokens x, the router W_r and the weights of its own experts, and
computes the routing of every token (router, per-expert top-C, token lists: tens of
microseconds). It runs the two expert GEMMs for its experts only, each row landing at
its token-major position in its Y. The owner of a token range then needs exactly the
rows of its tokens that each other rank computed; both sides list those rows from the
same token lists (``nmoe_ep_rows``), so sender and receiver agree on them without
exchanging anything. One all-to-all moves the rows, the owner unpacks them into its Y
and combines its token range in ascending expert order: its output rows equal a single
GPU's, bit for bit. The weight stream, the binding cost of the layer at small
capacities, is divided by the number of ranks.

Exchange sizes are static. A rank's experts own exactly E_g * Ce entries (expert choice:
every expert takes Ce = n_segments * C tokens), so the rows it owes any one rank number
at most E_g * Ce; every per-destination buffer has that many rows, filled in order and
padded (the row lists are padded with -1 on the device, and padded rows travel as
zeros). The split sizes of the all-to-all are therefore known on the host before the
layer runs, and the host never waits for a count: the whole layer, exchange included,
is enqueued without a synchronisation. The price is bytes: each rank sends (world - 1)
* E_g * Ce rows where the exact exchange would send about a world-th of that. With
``exact=True`` the counts are read back to the host first (one synchronisation per
call) and only the rows that exist travel.

``prepare`` and ``finish`` are the two halves around the exchange; ``forward`` runs them
with ``torch.distributed.all_to_all_single`` over NCCL (device buffers) or gloo (the
buffers staged through host memory).
"""

from __future__ import annotations

import ctypes as C

import torch

from . import _lib as L


def split_range(n: int, parts: int, index: int) -> tuple[int, int]:
    """[begin, end) of part `index` when n items are cut into `parts` contiguous parts
    whose sizes differ by at most one."""
    per, extra = divmod(n, parts)
    begin = index * per + min(index, extra)
    return begin, begin + per + (1 if index < extra else 0)


def exchange_plan(E: int, Ce: int, world: int, rank: int):
    """Static all-to-all split sizes, in rows, of the padded exchange: this rank sends
    E_g * Ce rows (its experts' entry count) to every other rank and receives E_r * Ce
    rows from every other rank r. Returns (send_splits, recv_splits), host lists in rank
    order, with 0 for this rank itself."""
    def cap(r):
        lo, hi = split_range(E, world, r)
        return (hi - lo) * Ce
    send = [0 if r == rank else cap(rank) for r in range(world)]
    recv = [0 if r == rank else cap(r) for r in range(world)]
    return send, recv


class Rank:
    """One rank's half-layer state between ``prepare`` and ``finish``."""

    def __init__(self, T, d, E, F, C_, world, rank, n_segments, dtype, workspace):
        self.T, self.d, self.E, self.F, self.C = T, d, E, F, C_
        self.world, self.rank = world, rank
        self.Ce = n_segments * C_
        self.dtype = dtype
        self.e_range = split_range(E, world, rank)
        self.t_range = split_range(T, world, rank)
        self.ws = workspace
        self.opts = dict(n_segments=n_segments, expert_begin=self.e_range[0],
                         expert_end=self.e_range[1], skip_combine=True)
        o = L.options(dtype=L._dt_code(dtype), **self.opts)
        y, tp, te = C.c_size_t(), C.c_size_t(), C.c_size_t()
        L._check(L.lib().nmoe_workspace_offsets(T, d, E, F, C_, C.byref(o), C.byref(y),
                                                C.byref(tp), C.byref(te)),
                 "nmoe_workspace_offsets")
        rows = E * self.Ce
        # Y is fp32: fp32 layers and the default split intermediates keep it so
        self.Y = workspace[y.value: y.value + rows * d * 4].view(torch.float32).view(rows, d)
        self.tok_ptr = workspace[tp.value: tp.value + (T + 1) * 4].view(torch.int32)
        self.tok_ent = workspace[te.value: te.value + rows * 4].view(torch.int32)
        self.send_splits, self.recv_splits = exchange_plan(E, self.Ce, world, rank)

    def rows(self, t_range, e_range, capacity, stream):
        """Token-major rows of tokens t_range whose expert lies in e_range, padded with -1
        to `capacity`, and their number (both on the device)."""
        dev = self.Y.device
        out = torch.empty(max(capacity, 1), dtype=torch.int32, device=dev)
        cnt = torch.empty(1, dtype=torch.int32, device=dev)
        L._check(L.lib().nmoe_ep_rows(self.tok_ptr.data_ptr(), self.tok_ent.data_ptr(),
                                      self.T, self.E, self.Ce, t_range[0], t_range[1],
                                      e_range[0], e_range[1], out.data_ptr(), capacity,
                                      cnt.data_ptr(), L._stream(stream)), "nmoe_ep_rows")
        return out, cnt


def _rows_copy(fn, src, rows, n, row_bytes, dst, stream):
    if n:
        L._check(fn(src.data_ptr(), rows.data_ptr(), n, row_bytes, dst.data_ptr(),
                    L._stream(stream)), "nmoe_rows_copy")


def prepare(x, W_r, W1, W3, W2, C_: int, E: int, world: int, rank: int, n_segments=1,
            workspace=None, stream=None, exact=False):
    """This rank's half: routing for every token, the expert GEMMs for its experts
    (W1, W3, W2 hold only those), and its rows packed for each destination rank.

    Returns (state, send buffer [sum of send splits, d] fp32, send splits, receive
    splits): host lists of rows in rank order (0 for this rank). By default the splits
    are the static padded sizes of ``exchange_plan`` and nothing waits for the device;
    with ``exact`` they are the true counts, read back to the host (one synchronisation).
    """
    T, d = x.shape
    F = W1.shape[2]
    if not 1 <= world <= E:
        raise ValueError("expert parallelism needs 1 <= world <= E")
    e_lo, e_hi = split_range(E, world, rank)
    if W1.shape[0] != e_hi - e_lo:
        raise ValueError(f"rank {rank} holds experts [{e_lo}, {e_hi}) but W1 has "
                         f"{W1.shape[0]}")
    opts = dict(n_segments=n_segments, expert_begin=e_lo, expert_end=e_hi, skip_combine=True)
    if workspace is None:
        workspace = torch.empty(L.workspace_size(T, d, E, F, C_, dtype=L._dt_code(x.dtype),
                                                 **opts),
                                dtype=torch.uint8, device=x.device)
    st = Rank(T, d, E, F, C_, world, rank, n_segments, x.dtype, workspace)
    o = L.options(dtype=L._dt_code(x.dtype), workspace=workspace, **opts)
    L._check(L.lib().nmoe_forward_ex(x.data_ptr(), W_r.data_ptr(), W1.data_ptr(),
                                     W3.data_ptr(), W2.data_ptr(), T, d, E, F, C_, None,
                                     L._stream(stream), C.byref(o)), "nmoe_forward_ex")
    # what I computed for each other owner; what each other rank computed for my tokens
    # (my own rows for my own tokens are already in my Y: nothing is listed for them)
    send, recv = [], []
    zero = torch.zeros(1, dtype=torch.int32, device=x.device)
    for r in range(world):
        if r == rank:
            send.append((None, zero))
            recv.append((None, zero))
            continue
        send.append(st.rows(split_range(T, world, r), st.e_range, st.send_splits[r], stream))
        recv.append(st.rows(st.t_range, split_range(E, world, r), st.recv_splits[r], stream))
    send_splits, recv_splits = list(st.send_splits), list(st.recv_splits)
    if exact:
        counts = torch.stack([c for _, c in send] + [c for _, c in recv]).view(-1)
        counts = counts.cpu().tolist()
        send_splits = [0 if r == rank else counts[r] for r in range(world)]
        recv_splits = [0 if r == rank else counts[world + r] for r in range(world)]
    st.send_rows = [rows for rows, _ in send]
    st.recv_rows = [rows for rows, _ in recv]
    st.recv_counts = recv_splits
    buf = torch.empty(sum(send_splits), d, dtype=torch.float32, device=x.device)
    at = 0
    for r in range(world):
        n = send_splits[r]
        _rows_copy(L.lib().nmoe_rows_gather, st.Y, st.send_rows[r], n, d * 4,
                   buf[at:at + n], stream)
        at += n
    return st, buf, send_splits, recv_splits


def finish(st: Rank, recv_buf, stream=None):
    """Unpacks the received rows into this rank's Y (padded rows are skipped) and
    combines its token range: returns out rows [t_end - t_begin, d] in the input dtype."""
    at = 0
    for r in range(st.world):
        n = st.recv_counts[r]
        _rows_copy(L.lib().nmoe_rows_scatter, recv_buf[at:at + n], st.recv_rows[r], n,
                   st.d * 4, st.Y, stream)
        at += n
    t0, t1 = st.t_range
    out = torch.empty(t1 - t0, st.d, dtype=st.dtype, device=st.Y.device)
    L._check(L.lib().nmoe_combine_tokens(st.Y.data_ptr(), st.tok_ptr.data_ptr(), st.T, st.d,
                                         t0, t1, L.NMOE_F32, L._dt_code(st.dtype),
                                         out.data_ptr(), L._stream(stream)),
             "nmoe_combine_tokens")
    return out


def all_to_all_rows(send, send_splits, recv_splits, group=None):
    """One all-to-all of row buffers with the given per-rank row splits. Over NCCL the
    device buffers travel directly; over gloo (host-only) they are staged through host
    memory. Returns the receive buffer on the send buffer's device."""
    import torch.distributed as dist
    d = send.shape[1]
    gloo = dist.get_backend(group) == "gloo"
    src = send.cpu() if gloo else send
    recv = torch.empty(sum(recv_splits), d, dtype=send.dtype, device=src.device)
    dist.all_to_all_single(recv, src, output_split_sizes=recv_splits,
                           input_split_sizes=send_splits, group=group)
    return recv.to(send.device) if gloo else recv


def forward(x, W_r, W1, W3, W2, C_: int, E: int, group=None, n_segments=1, workspace=None,
            exact=False):
    """The layer over the ranks of `group` (one GPU each): returns this rank's token range
    of the output (see split_range(T, world, rank))."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    st, send, send_splits, recv_splits = prepare(x, W_r, W1, W3, W2, C_, E, world, rank,
                                                 n_segments, workspace, exact=exact)
    recv = all_to_all_rows(send, send_splits, recv_splits, group)
    return finish(st, recv)
