"""The sharded convolution with the library's kernels, on one GPU: two ranks run as host threads
that exchange their halo rows through a shared in-process buffer (a stand-in for the NCCL
all-to-all, which needs one GPU per rank).  No kernel waits for another rank's kernel: the threads
meet only on the host, between launches, and every launch goes to the same stream.  The union of
the ranks' results must match the float64 oracle on the whole water-box graph."""

import math
import threading

import numpy as np
import pytest
import torch

import oracle
from mlip_message_passing_b200 import shard as S
from mlip_message_passing_b200 import workloads as W
from tests.conftest import rel_err

pytestmark = pytest.mark.gpu


class ThreadComm:
    """all-to-all between host threads of one process (device tensors stay on the device)."""

    def __init__(self, rank, world, shared):
        self.rank, self.world, self.shared = rank, world, shared

    def all_to_all(self, send, send_counts, recv_counts):
        box, bar = self.shared["box"], self.shared["barrier"]
        box[self.rank] = torch.split(send, list(send_counts))
        bar.wait()
        recv = torch.cat([box[s][self.rank] for s in range(self.world)], 0)
        assert recv.shape[0] == sum(recv_counts)
        bar.wait()  # every rank has taken its part before the next exchange reuses the box
        return recv


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_conv_threads_on_one_gpu(world):
    from mlip_message_passing_b200 import e3b
    n, mul, lx, ly, lo = 400, 64, 2, 3, 2
    g = W.graph_inputs(n, mul, lx, ly, lo, 5)
    order = np.argsort(g["dst"], kind="stable")
    src, dst = g["src"][order], g["dst"][order]
    vec, w = g["vec"][order], g["w"][order]
    row_ptr = np.concatenate([[0], np.cumsum(np.bincount(dst, minlength=n))])
    go = np.random.default_rng(6).standard_normal((n, W.out_dim(mul, lx, ly, lo))).astype(np.float32)
    s = 1 / math.sqrt(52)
    dev = torch.device("cuda", 0)
    shared = {"box": {}, "barrier": threading.Barrier(world)}
    results, errors = [None] * world, []

    def rank_main(rank):
        try:
            torch.cuda.set_device(dev)
            plan = e3b.Plan(W.irreps_str(mul, lx), W.sh_irreps(ly), lmax_out=lo)
            sh = S.ShardPlan(n, src, dst, row_ptr, rank, world)
            conv = S.ShardedConv(sh, ThreadComm(rank, world, shared), S.CudaBackend(plan, sh, dev))
            e = slice(sh.e_lo, sh.e_hi)
            x_own = torch.as_tensor(g["x"][sh.lo:sh.hi], device=dev)
            w_e, v_e = torch.as_tensor(w[e], device=dev), torch.as_tensor(vec[e], device=dev)
            out = conv.forward(x_own, w_e, v_e, s)
            dx, dy, dw = conv.backward(x_own, w_e, v_e, torch.as_tensor(go[sh.lo:sh.hi], device=dev), s)
            torch.cuda.synchronize()
            results[rank] = (sh, out.cpu().numpy(), dx.cpu().numpy(), dy.cpu().numpy(), dw.cpu().numpy())
        except BaseException as exc:  # reported below; the barrier is aborted so no thread waits
            errors.append(exc)
            shared["barrier"].abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not errors, errors
    e3b.device_status()
    q = oracle.make_plan(W.irreps_str(mul, lx), W.sh_irreps(ly), lmax_out=lo)
    Y = oracle.real_sh_all(ly, vec.astype(np.float64))
    ref = oracle.conv_forward(q, n, src, dst, g["x"], Y, w, s)
    rx, ry, rw = oracle.conv_backward(q, n, src, dst, g["x"], Y, w, go, s)
    out = np.zeros_like(ref)
    dx, dy, dw = np.zeros_like(rx), np.zeros_like(ry), np.zeros_like(rw)
    for sh, o, a, b, c in results:
        out[sh.lo:sh.hi], dx[sh.lo:sh.hi] = o, a
        dy[sh.e_lo:sh.e_hi], dw[sh.e_lo:sh.e_hi] = b, c
    assert rel_err(out, ref) <= 1e-5
    assert rel_err(dx, rx) <= 1e-5
    assert rel_err(dy, ry) <= 1e-5
    assert rel_err(dw, rw) <= 1e-5
