"""The expert-parallel exchange (ExpertParallelMoE) on CPU ranks: world size 2 over gloo.

The ranks run the module's real torch.distributed plumbing -- the row counts, the
all-to-all dispatch of tokens with their selections, the all-to-all return of the partial
rows and their per-token combine, or the all-gather / reduce-scatter pair -- with the device
steps replaced by CPU stand-ins written here from the oracle (routing, one expert's SwiGLU
FFN) and plain NumPy bookkeeping.  Each rank's output must equal the oracle's whole layer for
its tokens.  This checks the partition of the experts and the exchange; the device steps
themselves are checked against the oracle in test_expert_parallel_gpu.py."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class OracleOps:
    """CPU stand-ins for LibraryOps (fp32 tensors)."""

    def __init__(self, x_all_w, rank, world):
        from sparse_moe_layer_warp_b200.expert_parallel import expert_range

        self.w = x_all_w
        self.E, self.k = x_all_w["w_r"].shape[0], x_all_w["k"]
        self.e0, self.e1 = expert_range(self.E, rank, world)

    def route(self, x):
        from oracle import oracle_route, oracle_router_logits

        lg = oracle_router_logits(x.numpy(), self.w["w_r"])
        idx, gates = oracle_route(lg, self.w["b"], self.k)
        return torch.from_numpy(idx), torch.from_numpy(gates)

    def plan(self, idx, R):
        idx = idx.numpy()
        per = self.E // R
        need = np.stack([((idx >= q * per) & (idx < (q + 1) * per)).any(1) for q in range(R)], 1)
        bucket = np.where(need, np.arange(R)[None, :], R + np.arange(R)[None, :]).ravel()
        perm = np.argsort(bucket, kind="stable").astype(np.int32)
        cnt = np.bincount(bucket, minlength=2 * R).astype(np.int32)
        offsets = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int32)
        slot = np.empty_like(perm)
        slot[perm] = np.arange(len(perm), dtype=np.int32)
        return tuple(torch.from_numpy(a) for a in (cnt, offsets, perm, slot))

    def pack(self, x, idx, gates, perm, offsets, R, n_send):
        t = perm[:n_send].long() // R
        return x[t].contiguous(), idx[t].contiguous(), gates[t].contiguous()

    def partial(self, x, idx, gates, experts, shared):
        from oracle import oracle_expert_ffn

        w = self.w
        out = np.zeros((x.shape[0], x.shape[1]), np.float64)
        xn, idn, gn = x.numpy(), idx.numpy(), gates.numpy()
        for t in range(x.shape[0]):
            for j in range(self.k):
                e = int(idn[t, j])
                if experts[0] <= e < experts[1]:
                    le = e - self.e0  # this rank's weights: its experts, then the shared one
                    out[t] += w["rs"] * gn[t, j] * oracle_expert_ffn(
                        xn[t], w["wg"][le], w["wu"][le], w["wd"][le])
            if shared[0] <= t < shared[1]:
                s = self.e1 - self.e0
                out[t] += oracle_expert_ffn(xn[t], w["wg"][s], w["wu"][s], w["wd"][s])
        return torch.from_numpy(out.astype(np.float32))

    def combine(self, back, slot, offsets, shared, R, T):
        out = torch.zeros((T, self.w["w_r"].shape[1]), dtype=torch.float32)
        if back is not None:
            n = int(offsets[R])
            for t in range(T):
                for q in range(R):
                    r = int(slot[t * R + q])
                    if r < n:
                        out[t] += back[r]
        if shared is not None:
            out += shared
        return out


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, mode, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import oracle_moe_forward
        from sparse_moe_layer_warp_b200 import synth
        from sparse_moe_layer_warp_b200.expert_parallel import ExpertParallelMoE, expert_range

        wl = synth.WORKLOADS["tiny_fp32"].replace(T=24, d=64, E=8, k=3, f=32, seed=5,
                                                   routed_scale=1.5)
        inp = synth.make_inputs(wl)
        cv = synth.to_numpy_bits
        wg, wu, wd = cv(inp.w_gate), cv(inp.w_up), cv(inp.w_down)
        e0, e1 = expert_range(wl.E, rank, world)
        sl = lambda a: np.ascontiguousarray(np.concatenate([a[e0:e1], a[wl.E:]]))  # noqa: E731
        w = dict(w_r=cv(inp.w_router), b=cv(inp.bias), k=wl.k, rs=wl.routed_scale,
                 wg=sl(wg), wu=sl(wu), wd=sl(wd))
        ep = ExpertParallelMoE(OracleOps(w, rank, world), n_experts=wl.E, rank=rank,
                               world=world)
        # every rank its own tokens (uneven counts for the all-to-all)
        T_r = 12 if mode == "allgather" else (9 if rank == 0 else 15)
        x_all = cv(inp.x)
        lo = 0 if rank == 0 else (12 if mode == "allgather" else 9)
        x = torch.from_numpy(np.ascontiguousarray(x_all[lo:lo + T_r]))
        out = ep.forward(x, mode=mode).numpy().astype(np.float64)
        ref = oracle_moe_forward(x_all, w["w_r"], w["b"], wg, wu, wd, k=wl.k, n_shared=1,
                                 routed_scale=wl.routed_scale,
                                 tokens=np.arange(lo, lo + T_r, dtype=np.int32))[0]
        rms = float(np.sqrt(np.mean(ref ** 2)))
        q.put((rank, float(np.abs(out - ref).max() / rms)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode", ["alltoall", "allgather"])
def test_expert_parallel_exchange_world2(mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, mode, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = dict(q.get(timeout=5) for _ in range(2))
    # fp32 sums of the oracle's double expert outputs: far inside the fp32 parity bound
    assert max(res.values()) <= 1e-5, res
