"""Sharding one convolution graph over ranks (receiver ranges, halo exchange of x rows, reverse
exchange of grad_x partials), checked on the CPU: the plans of all ranks cover every edge exactly
once and agree on what they exchange, and gloo ranks whose local convolution is the float64
oracle reproduce the oracle on the whole graph.  The oracle stands in for the CUDA kernels only
here, to test the partition and exchange logic on a machine without a GPU."""

import math
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from mlip_message_passing_b200 import shard as S
from mlip_message_passing_b200 import workloads as W
from tests.conftest import rel_err


def graph(n=400, seed=3):
    g = W.graph_inputs(n, 4, 2, 3, 2, seed, dtype=np.float64, weights="none")
    dst, src, vec = g["dst"], g["src"], g["vec"]
    order = np.argsort(dst, kind="stable")  # global receiver order
    src, dst, vec = src[order], dst[order], vec[order]
    row_ptr = np.concatenate([[0], np.cumsum(np.bincount(dst, minlength=n))])
    rng = np.random.default_rng(seed + 1)
    return dict(n=n, src=src, dst=dst, vec=vec, row_ptr=row_ptr, x=g["x"], rng=rng)


@pytest.mark.parametrize("world", [1, 2, 3, 5])
def test_partition_balanced_and_covering(world):
    g = graph()
    b = S.receiver_partition(g["row_ptr"], world)
    assert b[0] == 0 and b[-1] == g["n"] and np.all(np.diff(b) >= 0)
    counts = np.diff(g["row_ptr"][b])
    E = int(g["row_ptr"][-1])
    deg_max = int(np.diff(g["row_ptr"]).max())
    assert counts.sum() == E
    assert np.all(np.abs(counts - E / world) <= deg_max)  # cut at receiver boundaries: within one row


@pytest.mark.parametrize("world", [2, 3])
def test_plans_cover_edges_and_agree_on_exchanges(world):
    g = graph()
    plans = [S.ShardPlan(g["n"], g["src"], g["dst"], g["row_ptr"], r, world) for r in range(world)]
    assert sum(p.e_hi - p.e_lo for p in plans) == g["src"].shape[0]
    for r, p in enumerate(plans):
        # local ids map back to the global edge list
        glob = np.concatenate([np.arange(p.lo, p.hi), p.halo])
        np.testing.assert_array_equal(glob[p.src_local], g["src"][p.e_lo:p.e_hi])
        np.testing.assert_array_equal(glob[p.dst_local], g["dst"][p.e_lo:p.e_hi])
        for s, q in enumerate(plans):
            # what s sends to r is what r receives from s, row for row
            assert q.send_counts[r] == p.recv_counts[s]
            got = q.lo + q.send_rows[r]
            want = p.halo[(p.halo >= q.lo) & (p.halo < q.hi)]
            np.testing.assert_array_equal(got, want)


class OracleBackend:
    """The local convolution of one rank computed by the float64 oracle (CPU tensors)."""

    def __init__(self, q, shard):
        self.q, self.sh = q, shard

    def forward(self, x_local, w, vec, scale):
        Y = oracle.real_sh_all(3, vec.numpy())
        out = oracle.conv_forward(self.q, self.sh.n_local, self.sh.src_local, self.sh.dst_local, x_local.numpy(), Y,
                                  w.numpy(), scale)
        return torch.as_tensor(out)

    def backward(self, x_local, w, vec, g_local, scale):
        Y = oracle.real_sh_all(3, vec.numpy())
        dx, dy, dw = oracle.conv_backward(self.q, self.sh.n_local, self.sh.src_local, self.sh.dst_local,
                                          x_local.numpy(), Y, w.numpy(), g_local.numpy(), scale)
        return torch.as_tensor(dx), torch.as_tensor(dy), torch.as_tensor(dw)

    def index(self, rows, device):
        return torch.as_tensor(np.asarray(rows, dtype=np.int64))

    def gather_rows(self, t, idx):
        return t[idx]

    def add_rows_(self, out, idx, t):
        out[idx] += t
        return out


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, result_path):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = graph()
        q = oracle.make_plan(W.irreps_str(4, 2), W.sh_irreps(3), lmax_out=2)
        rng = np.random.default_rng(11)
        w = rng.standard_normal((g["src"].shape[0], q.weight_numel))
        go = rng.standard_normal((g["n"], q.irreps_out.dim))
        sh = S.ShardPlan(g["n"], g["src"], g["dst"], g["row_ptr"], rank, world)
        conv = S.ShardedConv(sh, S.TorchComm(), OracleBackend(q, sh))
        s = 1 / math.sqrt(52)
        e = slice(sh.e_lo, sh.e_hi)
        x_own = torch.as_tensor(g["x"][sh.lo:sh.hi])
        out = conv.forward(x_own, torch.as_tensor(w[e]), torch.as_tensor(g["vec"][e]), s)
        dx, dy, dw = conv.backward(x_own, torch.as_tensor(w[e]), torch.as_tensor(g["vec"][e]),
                                   torch.as_tensor(go[sh.lo:sh.hi]), s)
        parts = [None] * world
        dist.all_gather_object(parts, (sh.lo, sh.hi, sh.e_lo, sh.e_hi, out.numpy(), dx.numpy(), dy.numpy(),
                                       dw.numpy()))
        if rank == 0:
            full_out = np.zeros((g["n"], q.irreps_out.dim))
            full_dx = np.zeros_like(g["x"])
            full_dy = np.zeros((g["src"].shape[0], 16))
            full_dw = np.zeros_like(w)
            for lo, hi, elo, ehi, o, a, b, c in parts:
                full_out[lo:hi], full_dx[lo:hi], full_dy[elo:ehi], full_dw[elo:ehi] = o, a, b, c
            Y = oracle.real_sh_all(3, g["vec"])
            ref = oracle.conv_forward(q, g["n"], g["src"], g["dst"], g["x"], Y, w, s)
            rx, ry, rw = oracle.conv_backward(q, g["n"], g["src"], g["dst"], g["x"], Y, w, go, s)
            errs = [rel_err(full_out, ref), rel_err(full_dx, rx), rel_err(full_dy, ry), rel_err(full_dw, rw)]
            np.save(result_path, np.array(errs))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_conv_on_gloo_ranks_equals_oracle(tmp_path, world):
    import torch.multiprocessing as mp
    path = str(tmp_path / "errs.npy")
    mp.start_processes(_rank_main, args=(world, _free_port(), path), nprocs=world, start_method="spawn")
    errs = np.load(path)
    assert np.all(errs <= 1e-12), errs
