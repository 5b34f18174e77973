"""Expert-parallel sparse-MoE layer: one rank's share of the layer and the token exchange
between ranks over ``torch.distributed`` (NCCL over NVLink / NVSwitch between GPUs).

"Step 3.5 Flash: Open Frontier-Level Intelligence with 11B Active Parameters" runs its MoE
layers expert-parallel (section 3: EP8 within a node) and balances the load across EP groups
of experts (section 2.2.2: the EP-group balance loss over G groups).  Here rank q of R holds
EP group q -- the E / R consecutive routed experts [q E / R, (q + 1) E / R), the grouping
``moe_router_stats`` uses for that loss -- plus the always-on shared expert, and the full
router (every rank routes its own tokens over all E experts).

Two exchanges, both deterministic:

* ``forward(x, mode="alltoall")`` (prefill-sized batches): route the rank's tokens, plan
  which tokens each rank needs (a token goes once to every rank that holds one of its
  experts), pack and send them with their selections (all-to-all), compute the received
  tokens' slots that fall in this rank's experts (fp32 partial rows), send those back
  (all-to-all) and add them per token in rank order, then the shared expert on the rank's own
  tokens, with one rounding;
* ``forward(x, mode="allgather")`` (decode-sized batches, the same token count on every
  rank): all-gather the tokens and their selections, compute every token's slots in this
  rank's experts plus the shared expert on the rank's own tokens (fp32), reduce-scatter the
  sums back to the tokens' ranks and round.

Every device step runs in ``libmoe_layer.so`` (``moe_route``, ``moe_ep_plan``,
``moe_ep_pack``, ``moe_forward_partial``, ``moe_ep_combine``); this module only moves
buffers between ranks.  The steps are reached through an ``ops`` object so that the exchange
logic can be exercised by processes without a GPU.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding


def expert_range(n_experts: int, rank: int, world: int):
    """Routed experts [begin, end) of EP group `rank` of `world` (consecutive ids)."""
    if n_experts % world != 0:
        raise ValueError(f"{n_experts} experts do not split evenly over {world} ranks")
    per = n_experts // world
    return rank * per, (rank + 1) * per


class LibraryOps:
    """The device steps of one rank, in the library (bf16 layer).

    Holds an expert-parallel handle (``moe_layer_init_ep``) over the rank's experts; its
    weight tensors hold those experts then the shared expert."""

    def __init__(self, w_router, router_bias, w_gate, w_up, w_down, *, n_experts, top_k,
                 max_tokens, rank, world, n_shared=1, routed_scale=1.0):
        e0, e1 = expert_range(n_experts, rank, world)
        if w_router.dtype != torch.bfloat16:
            raise ValueError("the expert-parallel layer runs the bf16 layer")
        d = int(w_router.shape[1])
        f = int(w_gate.shape[1])
        G = (e1 - e0) + int(n_shared)
        binding._expect(w_router, (n_experts, d), torch.bfloat16, "w_router")
        binding._expect(w_gate, (G, f, d), torch.bfloat16, "w_gate")
        binding._expect(w_up, (G, f, d), torch.bfloat16, "w_up")
        binding._expect(w_down, (G, d, f), torch.bfloat16, "w_down")
        if router_bias is not None:
            binding._expect(router_bias, (n_experts,), torch.float32, "router_bias")
        # a rank may receive every token of every rank
        self.cfg = binding.moe_config(int(max_tokens) * world, d, int(n_experts), int(top_k),
                                      f, int(n_shared), binding.MOE_BF16, float(routed_scale))
        self.tensors = (w_router, router_bias, w_gate, w_up, w_down)
        self.handle = binding.moe_layer_init_ep(self.cfg, e0, e1, *self.tensors)
        self.e0, self.e1 = e0, e1
        self.E, self.k, self.d = int(n_experts), int(top_k), d
        self.device = w_router.device
        self.ws = None

    def _ws(self, T):
        need = binding.moe_workspace_size(self.handle, max(T, 1))
        if self.ws is None or self.ws.numel() < need:
            self.ws = torch.empty(need, dtype=torch.uint8, device=self.device)
            binding.moe_workspace_init(self.handle, self.ws)
        return self.ws

    def route(self, x):
        T = int(x.shape[0])
        dev = self.device
        idx = torch.empty((T, self.k), dtype=torch.int32, device=dev)
        gates = torch.empty((T, self.k), dtype=torch.float32, device=dev)
        counts = torch.empty((self.E,), dtype=torch.int32, device=dev)
        offsets = torch.empty((self.E + 1,), dtype=torch.int32, device=dev)
        perm = torch.empty((T * self.k,), dtype=torch.int32, device=dev)
        slot = torch.empty((T, self.k), dtype=torch.int32, device=dev)
        binding.moe_route(self.handle, x, T, None, idx, gates, counts, offsets, perm, slot,
                          self._ws(T))
        return idx, gates

    def plan(self, idx, world):
        T = int(idx.shape[0])
        dev = self.device
        counts = torch.empty(2 * world, dtype=torch.int32, device=dev)
        offsets = torch.empty(2 * world + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(T * world, dtype=torch.int32, device=dev)
        slot = torch.empty(T * world, dtype=torch.int32, device=dev)
        binding.moe_ep_plan(self.handle, idx, T, world, counts, offsets, perm, slot,
                            self._ws(T))
        return counts, offsets, perm, slot

    def pack(self, x, idx, gates, perm, offsets, world, n_send):
        T = int(x.shape[0])
        rows = max(T * world, 1)
        xs = torch.empty((rows, self.d), dtype=x.dtype, device=self.device)
        ids = torch.empty((rows, self.k), dtype=torch.int32, device=self.device)
        gs = torch.empty((rows, self.k), dtype=torch.float32, device=self.device)
        binding.moe_ep_pack(self.handle, x, idx, gates, T, world, perm, offsets, xs, ids, gs)
        return xs[:n_send], ids[:n_send], gs[:n_send]

    def partial(self, x, idx, gates, experts, shared):
        T = int(x.shape[0])
        out = torch.empty((T, self.d), dtype=torch.float32, device=self.device)
        binding.moe_forward_partial(self.handle, x, T, idx, gates, experts[0], experts[1],
                                    shared[0], shared[1], out, self._ws(T))
        return out

    def combine(self, back, slot, offsets, shared, world, T):
        out = torch.empty((T, self.d), dtype=torch.bfloat16, device=self.device)
        binding.moe_ep_combine(self.handle, back, slot, offsets, shared, T, world, out)
        return out

    def close(self):
        if self.handle is not None:
            binding.moe_layer_destroy(self.handle)
            self.handle = None


class ExpertParallelMoE:
    """One rank of an expert-parallel layer: ``forward`` exchanges tokens with the other
    ranks of `group` (default: the whole world) and returns this rank's outputs."""

    def __init__(self, ops, *, n_experts, rank, world, group=None):
        self.ops = ops
        self.E = int(n_experts)
        self.rank, self.world = int(rank), int(world)
        self.group = group
        self.experts = expert_range(self.E, self.rank, self.world)

    def forward(self, x, mode="alltoall"):
        if mode == "alltoall":
            return self._forward_alltoall(x)
        if mode == "allgather":
            return self._forward_allgather(x)
        raise ValueError(mode)

    # -------------------------------------------------------------- dispatch / combine
    def _forward_alltoall(self, x):
        ops, R = self.ops, self.world
        T = int(x.shape[0])
        idx, gates = ops.route(x)
        counts, offsets, perm, slot = ops.plan(idx, R)
        send = [int(v) for v in counts[:R].tolist()]  # rows per destination (host copy)
        n_send = sum(send)
        xs, ids, gs = ops.pack(x, idx, gates, perm, offsets, R, n_send)
        # the row counts each rank will receive
        sc = torch.tensor(send, dtype=torch.int64, device=x.device)
        rc = torch.empty_like(sc)
        dist.all_to_all_single(rc, sc, group=self.group)
        recv = [int(v) for v in rc.tolist()]
        n_recv = sum(recv)
        xr = torch.empty((n_recv, x.shape[1]), dtype=x.dtype, device=x.device)
        ir = torch.empty((n_recv, ids.shape[1]), dtype=ids.dtype, device=x.device)
        gr = torch.empty((n_recv, gs.shape[1]), dtype=gs.dtype, device=x.device)
        pending = [dist.all_to_all_single(xr, xs, recv, send, group=self.group, async_op=True),
                   dist.all_to_all_single(ir, ids, recv, send, group=self.group, async_op=True),
                   dist.all_to_all_single(gr, gs, recv, send, group=self.group, async_op=True)]
        # the shared expert on this rank's own tokens needs nothing from the exchange: it runs
        # while the rows are in flight (on the compute stream, beside the collectives' own)
        shared = ops.partial(x, idx, gates, (self.experts[0], self.experts[0]), (0, T))
        for work in pending:
            work.wait()
        # the received tokens' slots in this rank's experts (no shared expert here)
        part = ops.partial(xr, ir, gr, self.experts, (0, 0))
        back = torch.empty((n_send, x.shape[1]), dtype=torch.float32, device=x.device)
        dist.all_to_all_single(back, part, send, recv, group=self.group)
        # the per-token sum in rank order
        return ops.combine(back, slot, offsets, shared, R, T)

    def _forward_allgather(self, x):
        ops, R = self.ops, self.world
        T = int(x.shape[0])
        idx, gates = ops.route(x)
        xa = torch.empty((R * T, x.shape[1]), dtype=x.dtype, device=x.device)
        ia = torch.empty((R * T, idx.shape[1]), dtype=idx.dtype, device=x.device)
        ga = torch.empty((R * T, gates.shape[1]), dtype=gates.dtype, device=x.device)
        dist.all_gather_into_tensor(xa, x.contiguous(), group=self.group)
        dist.all_gather_into_tensor(ia, idx.contiguous(), group=self.group)
        dist.all_gather_into_tensor(ga, gates.contiguous(), group=self.group)
        # every token's slots in this rank's experts, the shared expert on its own tokens
        part = ops.partial(xa, ia, ga, self.experts, (self.rank * T, (self.rank + 1) * T))
        mine = torch.empty((T, x.shape[1]), dtype=torch.float32, device=x.device)
        dist.reduce_scatter_tensor(mine, part, op=dist.ReduceOp.SUM, group=self.group)
        return ops.combine(None, None, None, mine, R, T)
