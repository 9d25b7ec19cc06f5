"""One convolution graph sharded over ranks (one process per GPU).

The convolution sums messages into receivers through the receiver CSR (E3J summary, section
E.2.2), so a contiguous range of receivers, with all of its in-edges, is a self-contained piece of
work.  Rank r owns

* receivers [lo_r, hi_r): their node rows (x, out, grad_out, grad_x) live on rank r;
* the in-edges of those receivers: positions [row_ptr[lo_r], row_ptr[hi_r]) of the global edge list
  in receiver order, so every per-edge array (weights, edge vectors, grad_y, grad_w) is a
  contiguous slice that never leaves the rank.

The ranges split the edges evenly (integer arithmetic on row_ptr, bit-exact on every rank).  What
crosses ranks is the node rows of the senders outside the own range (the halo):

* forward: each rank receives the x rows of its halo senders from their owners (one all-to-all),
  runs the convolution on its local graph (owned receivers first, then halo senders), and keeps
  the owned output rows -- no reduction;
* backward: grad_out rows are already local (they belong to the owned receivers); the local
  backward gives grad_x for owned and halo senders; the halo rows go back to their owners (the
  reverse all-to-all), which add them to their own rows in ascending source-rank order, so the
  result is deterministic.

Every rank holds the (integer) global topology and derives every other rank's plan from it, so no
metadata is exchanged.  The communicator and the compute backend are injected: `TorchComm` (NCCL
between GPUs, or gloo) with `CudaBackend` (this library's kernels) is the product path; tests run
the same partition and exchange logic with other backends.
"""

import numpy as np


def receiver_partition(row_ptr, world):
    """Boundaries b[0..world] of contiguous receiver ranges with about E/world in-edges each:
    rank r owns receivers [b[r], b[r+1]).  row_ptr: the global receiver CSR [N + 1]."""
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    n = row_ptr.shape[0] - 1
    e = int(row_ptr[-1])
    b = np.zeros(world + 1, dtype=np.int64)
    for r in range(1, world):
        target = (e * r) // world
        # first receiver whose in-edges start at or after the target position
        b[r] = int(np.searchsorted(row_ptr[:n + 1], target, side="left"))
        b[r] = min(max(b[r], b[r - 1]), n)
    b[world] = n
    return b


class ShardPlan:
    """Host-side plan of one rank (numpy, integer-only).

    src, dst: global int arrays in global receiver order (dst non-decreasing); row_ptr: the
    global receiver CSR.  Local node numbering: owned receivers 0 .. n_own-1 (global lo .. hi-1),
    then the halo senders in ascending global id."""

    def __init__(self, n_nodes, src, dst, row_ptr, rank, world):
        src = np.asarray(src, dtype=np.int64)
        dst = np.asarray(dst, dtype=np.int64)
        row_ptr = np.asarray(row_ptr, dtype=np.int64)
        if np.any(np.diff(dst) < 0):
            raise ValueError("edges must be in receiver order (dst non-decreasing)")
        self.n_nodes, self.rank, self.world = int(n_nodes), int(rank), int(world)
        self.bounds = receiver_partition(row_ptr, world)
        b = self.bounds
        self.lo, self.hi = int(b[rank]), int(b[rank + 1])
        self.n_own = self.hi - self.lo
        self.e_lo, self.e_hi = int(row_ptr[self.lo]), int(row_ptr[self.hi])
        owner = np.searchsorted(b[1:], np.arange(self.n_nodes), side="right")  # owner rank of each node
        self.owner = owner

        def halo_of(r):
            s = src[int(row_ptr[b[r]]):int(row_ptr[b[r + 1]])]
            h = np.unique(s)
            return h[(h < b[r]) | (h >= b[r + 1])]

        halos = [halo_of(r) for r in range(world)]
        self.halo = halos[rank]
        self.n_local = self.n_own + self.halo.shape[0]
        # local ids: owned receivers first, then halo senders (ascending global id)
        local_of = np.full(self.n_nodes, -1, dtype=np.int64)
        local_of[self.lo:self.hi] = np.arange(self.n_own)
        local_of[self.halo] = self.n_own + np.arange(self.halo.shape[0])
        es = src[self.e_lo:self.e_hi]
        self.src_local = local_of[es].astype(np.int32)
        self.dst_local = (dst[self.e_lo:self.e_hi] - self.lo).astype(np.int32)
        # forward exchange: rows of my owned x that rank r needs (owned-local row ids), in ascending
        # global id; and how many rows I receive from each rank (my halo, grouped by owner)
        self.send_rows = []
        for r in range(world):
            h = halos[r]
            mine = h[(h >= self.lo) & (h < self.hi)] if r != rank else h[:0]
            self.send_rows.append((mine - self.lo).astype(np.int64))
        self.recv_counts = [int(np.count_nonzero(owner[self.halo] == s)) for s in range(world)]
        self.send_counts = [int(v.shape[0]) for v in self.send_rows]


class TorchComm:
    """all-to-all with uneven splits through torch.distributed (NCCL for device tensors, gloo for
    host tensors).  Rows of a 2-D tensor are the units."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group

    def all_to_all(self, send, send_counts, recv_counts):
        import torch
        out = torch.empty((sum(recv_counts),) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
        self.dist.all_to_all_single(out, send.contiguous(), list(recv_counts), list(send_counts), group=self.group)
        return out


class CudaBackend:
    """The convolution of one rank's local graph with this library's kernels (e3b)."""

    def __init__(self, plan, shard, device, sh_norm="component"):
        import torch
        from . import e3b
        self.e3b, self.plan, self.sh_norm = e3b, plan, sh_norm
        src = torch.as_tensor(shard.src_local, device=device)
        dst = torch.as_tensor(shard.dst_local, device=device)
        # the local edges are already in receiver order: the local CSR keeps their order
        self.graph = e3b.Graph(shard.n_local, src, dst)

    def forward(self, x_local, w, vec, scale):
        return self.e3b.conv_forward(self.plan, self.graph, x_local, w, edge_vec=vec, sh_norm=self.sh_norm,
                                     out_scale=scale)

    def backward(self, x_local, w, vec, g_local, scale):
        return self.e3b.conv_backward(self.plan, self.graph, x_local, w, g_local, edge_vec=vec, sh_norm=self.sh_norm,
                                      out_scale=scale)

    def index(self, rows, device):
        import torch
        return torch.as_tensor(np.asarray(rows, dtype=np.int32), device=device)

    def gather_rows(self, t, idx):
        return self.e3b.gather_rows(idx, t.contiguous())

    def add_rows_(self, out, idx, t):
        return self.e3b.add_rows_(out, idx, t.contiguous())


class ShardedConv:
    """Forward and backward of the convolution over one rank's shard (see the module docstring).

    Node arrays passed in and returned are the rank's owned rows ([n_own, .]); edge arrays are
    the rank's slice [e_lo, e_hi) of the global receiver-ordered edge list."""

    def __init__(self, shard, comm, backend):
        self.shard, self.comm, self.backend = shard, comm, backend
        self._idx = {}

    def _index(self, key, rows, device):
        if key not in self._idx:
            self._idx[key] = self.backend.index(rows, device)
        return self._idx[key]

    def gather_halo(self, x_owned):
        """x rows of the local graph: the owned rows, then the halo senders' rows from their owners."""
        import torch
        sh = self.shard
        if sh.world == 1:
            return x_owned
        rows = np.concatenate(sh.send_rows) if sh.send_rows else np.zeros(0, np.int64)
        send = self.backend.gather_rows(x_owned, self._index("send", rows, x_owned.device))
        recv = self.comm.all_to_all(send, sh.send_counts, sh.recv_counts)
        return torch.cat([x_owned, recv], dim=0)

    def forward(self, x_owned, w, vec, scale):
        x_local = self.gather_halo(x_owned)
        return self.backend.forward(x_local, w, vec, scale)[:self.shard.n_own]

    def backward(self, x_owned, w, vec, g_owned, scale):
        """(grad_x of the owned rows, grad_y and grad_w of the rank's edges)."""
        import torch
        sh = self.shard
        x_local = self.gather_halo(x_owned)
        g_local = g_owned if sh.n_local == sh.n_own else torch.cat(
            [g_owned, g_owned.new_zeros((sh.n_local - sh.n_own,) + tuple(g_owned.shape[1:]))], 0)
        dx, dy, dw = self.backend.backward(x_local, w, vec, g_local, scale)
        if sh.world == 1:
            return dx, dy, dw
        # halo partials go back to their owners (the reverse of the forward exchange)
        part = self.comm.all_to_all(dx[sh.n_own:], sh.recv_counts, sh.send_counts)
        dx_own = dx[:sh.n_own].contiguous()
        off = 0
        for s in range(sh.world):  # fixed order: ascending source rank
            k = sh.send_counts[s]
            if k:
                self.backend.add_rows_(dx_own, self._index(("add", s), sh.send_rows[s], dx.device), part[off:off + k])
            off += k
        return dx_own, dy, dw
