"""Expert-parallel layer on one GPU: the library's device steps of the split layer
(moe_forward_partial, moe_ep_plan, moe_ep_pack, moe_ep_combine, moe_layer_init_ep), with the
ranks' exchanges emulated in this process (one GPU holds every rank's buffers; no rank ever
waits on another).  Checked against the full forward and the CPU oracle."""
import numpy as np
import pytest
import torch

from sparse_moe_layer_warp_b200 import binding, synth
from sparse_moe_layer_warp_b200.expert_parallel import LibraryOps, expert_range
from tests.helpers import compare_layer, make_layer

pytestmark = pytest.mark.gpu

CASES = [
    dict(T=40, d=256, E=32, k=4, f=128, seed=1),                    # one-CTA, gathered rows
    dict(T=300, d=512, E=32, k=8, f=256, seed=2),                   # one-CTA, sorted copy
    dict(T=700, d=768, E=8, k=4, f=512, seed=6),                    # CTA pairs
    dict(T=257, d=256, E=48, k=6, f=256, seed=3, bias="zipf"),      # skewed, empty experts
]


def _inputs(kw):
    w = synth.WORKLOADS["tiny_fp32"].replace(dtype="bf16", **kw)
    return w, synth.make_inputs(w, device="cuda")


def _partial(layer, x, e0, e1, s0, s1, idx=None, gates=None):
    T = x.shape[0]
    out = torch.full((T, x.shape[1]), float("nan"), dtype=torch.float32, device="cuda")
    binding.moe_forward_partial(layer.handle, x, T, idx, gates, e0, e1, s0, s1, out,
                                layer.workspace(T))
    return out


def _round(layer, s):
    T = s.shape[0]
    out = torch.empty((T, s.shape[1]), dtype=torch.bfloat16, device="cuda")
    binding.moe_ep_combine(layer.handle, None, None, None, s, T, 1, out)
    return out


@pytest.mark.parametrize("kw", CASES)
@pytest.mark.parametrize("R", [2, 4])
@pytest.mark.parametrize("gather", [1, 2])
def test_partials_over_expert_slices_sum_to_the_layer(cuda_ok, kw, R, gather):
    """Partials of a partition of the experts (the shared expert in one of them) add up to
    the layer: within fp32 reordering of the forward's sum, and within the parity bound of
    the oracle.  gather = 2: CTA-pair partials write the sorted copy inside the up GEMM,
    skipping the rows of other ranks' experts."""
    w, inp = _inputs(kw)
    layer = make_layer(inp)
    layer.set_option(binding.MOE_OPTION_ROW_GATHER_IN_GEMM, gather)
    full = layer.forward(inp.x)
    T = w.T
    tot = torch.zeros((T, w.d), dtype=torch.float32, device="cuda")
    for q in range(R):
        e0, e1 = expert_range(w.E, q, R)
        tot += _partial(layer, inp.x, e0, e1, 0, T if q == 0 else 0)
    out = _round(layer, tot)
    r = layer.route(x=inp.x)
    torch.cuda.synchronize()
    # the same per-row expert outputs, summed in another fp32 order: at most a few bf16 ulps
    diff = (out.float() - full.float()).abs()
    assert (diff <= 2.0 ** -6 * full.float().abs() + 1e-3).all(), diff.max().item()
    compare_layer(inp, out, r["idx"].cpu().numpy())
    assert layer.device_status() == 0


def test_partial_with_given_selection_equals_own_routing(cuda_ok):
    w, inp = _inputs(CASES[1])
    layer = make_layer(inp)
    r = layer.route(x=inp.x)
    a = _partial(layer, inp.x, 8, 24, 5, 200)
    b = _partial(layer, inp.x, 8, 24, 5, 200, r["idx"], r["gates"])
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    # nothing in range and no shared tokens: exact zeros; shared only: the shared expert
    z = _partial(layer, inp.x, 8, 8, 0, 0, r["idx"], r["gates"])
    torch.cuda.synchronize()
    assert (z == 0).all()
    assert layer.device_status() == 0


def test_ep_plan_matches_reference_bit_exact(cuda_ok):
    w, inp = _inputs(CASES[3])
    layer = make_layer(inp)
    r = layer.route(x=inp.x)
    T, R = w.T, 4
    ops_counts = torch.empty(2 * R, dtype=torch.int32, device="cuda")
    offsets = torch.empty(2 * R + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * R, dtype=torch.int32, device="cuda")
    slot = torch.empty(T * R, dtype=torch.int32, device="cuda")
    binding.moe_ep_plan(layer.handle, r["idx"], T, R, ops_counts, offsets, perm, slot,
                        layer.workspace(T))
    torch.cuda.synchronize()
    idx = r["idx"].cpu().numpy()
    per = w.E // R
    need = np.stack([((idx >= q * per) & (idx < (q + 1) * per)).any(1) for q in range(R)], 1)
    # pair (t, q) -> bucket q (sent to q) or R + q (nothing for q); ascending t per bucket
    bucket = np.where(need, np.arange(R)[None, :], R + np.arange(R)[None, :]).ravel()
    order = np.argsort(bucket, kind="stable")
    cnt = np.bincount(bucket, minlength=2 * R)
    assert (ops_counts.cpu().numpy() == cnt).all()
    assert (offsets.cpu().numpy() == np.concatenate([[0], np.cumsum(cnt)])).all()
    assert (perm.cpu().numpy() == order).all()
    inv = np.empty_like(order)
    inv[order] = np.arange(len(order))
    assert (slot.cpu().numpy() == inv).all()


@pytest.mark.parametrize("kw", CASES[1:])
@pytest.mark.parametrize("R", [2, 3])
def test_emulated_alltoall_exchange_matches_oracle(cuda_ok, kw, R):
    """Every rank: its own expert-parallel handle over sliced weights (its experts, then the
    shared expert), its own tokens.  The all-to-all exchange of ExpertParallelMoE is emulated
    by slicing the ranks' send buffers; outputs against the oracle."""
    kw = dict(kw)
    w, inp = _inputs(kw)
    if w.E % R:
        pytest.skip("experts do not split over the ranks")
    T = w.T
    bounds = [T * q // R for q in range(R + 1)]
    ranks = []
    for q in range(R):
        e0, e1 = expert_range(w.E, q, R)
        sl = lambda t: torch.cat([t[e0:e1], t[w.E:]]).contiguous()  # noqa: E731
        ops = LibraryOps(inp.w_router, inp.bias, sl(inp.w_gate), sl(inp.w_up), sl(inp.w_down),
                         n_experts=w.E, top_k=w.k, max_tokens=T, rank=q, world=R,
                         n_shared=w.n_shared, routed_scale=w.routed_scale)
        ranks.append(ops)
    xs = [inp.x[bounds[q]:bounds[q + 1]].contiguous() for q in range(R)]
    # each rank: route, plan, pack
    st = []
    for q, ops in enumerate(ranks):
        idx, gates = ops.route(xs[q])
        counts, offsets, perm, slot = ops.plan(idx, R)
        send = [int(v) for v in counts[:R].tolist()]
        xb, ib, gb = ops.pack(xs[q], idx, gates, perm, offsets, R, sum(send))
        st.append(dict(idx=idx, gates=gates, offsets=offsets, slot=slot, send=send, xb=xb,
                       ib=ib, gb=gb))
    # the exchange: rank p receives from every rank q its block for p, in rank order
    back_parts = [[None] * R for _ in range(R)]
    for p, ops in enumerate(ranks):
        blocks = []
        for q in range(R):
            o = sum(st[q]["send"][:p])
            n = st[q]["send"][p]
            blocks.append((q, o, n))
        xr = torch.cat([st[q]["xb"][o:o + n] for q, o, n in blocks])
        ir = torch.cat([st[q]["ib"][o:o + n] for q, o, n in blocks])
        gr = torch.cat([st[q]["gb"][o:o + n] for q, o, n in blocks])
        part = ops.partial(xr, ir, gr, ops_range(ops), (0, 0)) if xr.shape[0] else \
            torch.empty((0, w.d), dtype=torch.float32, device="cuda")
        o2 = 0
        for q, _, n in blocks:
            back_parts[q][p] = part[o2:o2 + n]
            o2 += n
    outs = []
    for q, ops in enumerate(ranks):
        back = torch.cat(back_parts[q]) if sum(st[q]["send"]) else None
        Tq = xs[q].shape[0]
        shared = ops.partial(xs[q], st[q]["idx"], st[q]["gates"],
                             (ops.e0, ops.e0), (0, Tq))
        outs.append(ops.combine(back, st[q]["slot"], st[q]["offsets"], shared, R, Tq))
    out = torch.cat(outs)
    full = make_layer(inp).route(x=inp.x)
    torch.cuda.synchronize()
    compare_layer(inp, out, full["idx"].cpu().numpy())
    for ops in ranks:
        ops.close()


def ops_range(ops):
    return (ops.e0, ops.e1)


def test_slice_handle_refuses_whole_layer_calls(cuda_ok):
    w, inp = _inputs(CASES[0])
    e0, e1 = expert_range(w.E, 1, 4)
    sl = lambda t: torch.cat([t[e0:e1], t[w.E:]]).contiguous()  # noqa: E731
    ops = LibraryOps(inp.w_router, inp.bias, sl(inp.w_gate), sl(inp.w_up), sl(inp.w_down),
                     n_experts=w.E, top_k=w.k, max_tokens=w.T, rank=1, world=4)
    ws = ops._ws(w.T)
    out = torch.empty_like(inp.x)
    with pytest.raises(binding.MoEError) as e:
        binding.moe_forward(ops.handle, inp.x, w.T, out, ws)
    assert e.value.status == binding.MOE_ERR_UNSUPPORTED
    p = torch.empty((w.T, w.d), dtype=torch.float32, device="cuda")
    with pytest.raises(binding.MoEError) as e:  # experts outside the handle's range
        binding.moe_forward_partial(ops.handle, inp.x, w.T, None, None, 0, e1, 0, 0, p, ws)
    assert e.value.status == binding.MOE_ERR_INVALID_ARG
    ops.close()


@pytest.mark.parametrize("kw", CASES)
def test_shared_expert_token_subranges(cuda_ok, kw):
    """The shared expert on a token range that starts inside the batch (the all-gather
    exchange gives each rank its own tokens' shared rows): three partials whose shared ranges
    partition the tokens, one of them also holding every routed expert, sum to the layer."""
    w, inp = _inputs(kw)
    layer = make_layer(inp)
    T = w.T
    s0, s1 = T // 3, (2 * T) // 3 + 1
    tot = _partial(layer, inp.x, 0, w.E, s0, s1)
    tot += _partial(layer, inp.x, 0, 0, 0, s0)
    tot += _partial(layer, inp.x, w.E, w.E, s1, T)
    out = _round(layer, tot)
    r = layer.route(x=inp.x)
    torch.cuda.synchronize()
    compare_layer(inp, out, r["idx"].cpu().numpy())
    assert layer.device_status() == 0


@pytest.mark.parametrize("kw", [CASES[0], CASES[2]])
@pytest.mark.parametrize("R", [2, 4])
def test_emulated_allgather_exchange_matches_oracle(cuda_ok, kw, R):
    """ExpertParallelMoE's all-gather exchange emulated on one GPU: every rank (its own
    handle over sliced weights) computes all ranks' tokens in its experts plus the shared
    expert on its own tokens; the per-token sum of the ranks' partials (the reduce-scatter)
    is rounded by moe_ep_combine."""
    w, inp = _inputs(kw)
    if w.E % R or w.T % R:
        pytest.skip("experts or tokens do not split over the ranks")
    T = w.T
    Tr = T // R
    ranks = []
    for q in range(R):
        e0, e1 = expert_range(w.E, q, R)
        sl = lambda t: torch.cat([t[e0:e1], t[w.E:]]).contiguous()  # noqa: E731
        ranks.append(LibraryOps(inp.w_router, inp.bias, sl(inp.w_gate), sl(inp.w_up),
                                sl(inp.w_down), n_experts=w.E, top_k=w.k, max_tokens=Tr,
                                rank=q, world=R, n_shared=w.n_shared,
                                routed_scale=w.routed_scale))
    # each rank routes its own tokens; the all-gather concatenates them in rank order
    sel = [ranks[q].route(inp.x[q * Tr:(q + 1) * Tr].contiguous()) for q in range(R)]
    ia = torch.cat([s[0] for s in sel])
    ga = torch.cat([s[1] for s in sel])
    tot = torch.zeros((T, w.d), dtype=torch.float32, device="cuda")
    for q, ops in enumerate(ranks):
        tot += ops.partial(inp.x, ia, ga, (ops.e0, ops.e1), (q * Tr, (q + 1) * Tr))
    out = torch.cat([ranks[q].combine(None, None, None, tot[q * Tr:(q + 1) * Tr].contiguous(),
                                      R, Tr) for q in range(R)])
    full = make_layer(inp).route(x=inp.x)
    torch.cuda.synchronize()
    compare_layer(inp, out, full["idx"].cpu().numpy())
    for ops in ranks:
        ops.close()
