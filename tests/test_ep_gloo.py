"""Expert parallelism: the dispatch/combine index arithmetic and the
reassembled layer, on CPU.

The exchange (group_limited_routed_moe_b200.ep) runs here with the float64
oracle standing in for the two library calls it makes on GPUs (the owner's
grouped expert FFN and the source's combine), passed explicitly as
``compute`` / ``combine``:
  - the plan alone for W = 8: every token reaches at most 4 ranks (the group
    limit), rows go destination-major and token-ascending, and every slot
    comes back to exactly one place;
  - W = 2, 4, 8 ranks run in lockstep by one process, and W = 2 real gloo
    ranks (torch.distributed all-to-all): each rank receives exactly the rows
    of every token that routed to one of its experts, with the right local
    ids, and the layer output reassembled from the returned rows equals the
    oracle's layer on the rank's own tokens (same float64 arithmetic in
    another summation order: relative 1e-12);
  - edge cases: an empty batch, one rank holding every expert, and a rank
    without tokens that still serves the rows routed to its experts.
"""
import os

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle as O
from group_limited_routed_moe_b200 import ep, synth

T_PER_RANK = 6


def _tokens(rank):
    tok = synth.make_tokens(T_PER_RANK, 20 + rank)
    rr = O.route(tok.logits, tok.bias)
    return tok, rr


class _OracleExperts:
    """Host weights of the experts on demand (float64 values)."""

    def __init__(self):
        self.cache = {}

    def get(self, e):
        if e not in self.cache:
            w = synth.layer_weights_np(0, 0, [e])
            self.cache[e] = tuple(O.bf16_bits_to_f64(m[0]) for m in w)
        return self.cache[e]


def _oracle_compute(rank, world, experts):
    n_loc = ep.experts_per_rank(world)

    def compute(recv_x, recv_local):
        x = O.bf16_bits_to_f64(recv_x.view(torch.int16).numpy().view(np.uint16))
        loc = recv_local.numpy()
        rows, slots = np.nonzero(loc >= 0)         # (row, slot) order
        y = np.empty((len(rows), ep.HIDDEN))
        for i, (r, j) in enumerate(zip(rows, slots)):
            wg, wu, wd = experts.get(rank * n_loc + int(loc[r, j]))
            y[i] = O.expert_ffn(x[r:r + 1], wg, wu, wd)[0]
        return torch.from_numpy(y)
    return compute


def _oracle_combine(y_back, topk_w, ret_index, residual, out):
    y = y_back.numpy()
    w = np.asarray(topk_w)
    idx = ret_index.numpy().reshape(-1, ep.TOPK)
    res = np.zeros((w.shape[0], ep.HIDDEN))
    for s in range(ep.TOPK):                      # slot order, as the GPU combine
        res += w[:, s:s + 1] * y[idx[:, s]]
    return torch.from_numpy(res)


def _expected_layer(tok, rr):
    ex = np.unique(rr.topk_idx)
    ws = synth.layer_weights_np(0, 0, ex)
    import dataclasses
    rc = dataclasses.replace(rr, topk_idx=np.searchsorted(ex, rr.topk_idx))
    return O.moe_layer(tok.x_bits, tok.logits, tok.bias, *ws, route_result=rc)


def _expected_recv(rank, world):
    """Rows rank receives: (source rank, token) of every token with an expert
    in its slice, source-major then token-ascending, with local slot ids."""
    n_loc = ep.experts_per_rank(world)
    rows, local = [], []
    for s in range(world):
        tok, rr = _tokens(s)
        for t in range(T_PER_RANK):
            own = (rr.topk_idx[t] // n_loc) == rank
            if own.any():
                rows.append(tok.x_bits[t])
                local.append(np.where(own, rr.topk_idx[t] - rank * n_loc, -1))
    if not rows:
        return np.zeros((0, ep.HIDDEN), np.uint16), np.zeros((0, ep.TOPK), np.int64)
    return np.stack(rows), np.stack(local)


def test_plan_group_limit_and_layout():
    rng = np.random.default_rng(5)
    lg = rng.standard_normal((300, 128)).astype(np.float32)
    rr = O.route(lg, None)
    idx = torch.from_numpy(rr.topk_idx)
    W = 8
    p = ep.plan_dispatch(idx, W)
    owner = rr.topk_idx // 16
    fan = np.array([len(set(o)) for o in owner])
    assert fan.max() <= 4 and np.array_equal(p.send_counts.numpy(),
                                             [(owner == d).any(1).sum() for d in range(W)])
    # destination-major, token-ascending rows with the right local ids
    k = 0
    for d in range(W):
        for t in range(300):
            if (owner[t] == d).any():
                assert p.send_tok[k] == t
                np.testing.assert_array_equal(
                    p.send_local[k].numpy(), np.where(owner[t] == d, rr.topk_idx[t] - 16 * d, -1))
                k += 1
    assert k == p.send_tok.numel()
    # every (token, slot) has one place in the returned rows, owner-major, item order
    ri = p.ret_index.numpy()
    assert np.array_equal(np.sort(ri), np.arange(300 * 8))
    flat = owner.reshape(-1)
    assert np.array_equal(np.argsort(ri), np.argsort(flat, kind="stable"))
    assert np.array_equal(p.ret_counts.numpy(), np.bincount(flat, minlength=W))


@pytest.mark.parametrize("world", [2, 4, 8])
def test_in_process_ranks_reassemble_the_layer(world):
    experts = _OracleExperts()
    layers, xs, idxs, ws, refs = [], [], [], [], []
    for r in range(world):
        tok, rr = _tokens(r)
        layers.append(ep.ExpertParallelMoE(r, world, compute=_oracle_compute(r, world, experts),
                                           combine=_oracle_combine))
        xs.append(torch.from_numpy(tok.x_bits.view(np.int16)).view(torch.bfloat16))
        idxs.append(torch.from_numpy(rr.topk_idx))
        ws.append(rr.topk_w)
        refs.append(_expected_layer(tok, rr))
    outs = ep.forward_in_process(layers, xs, idxs, ws)
    for r in range(world):
        assert O.rel_l2(outs[r].numpy(), refs[r]) <= 1e-12


def _gloo_rank(rank, world, port, q):
    try:
        import torch.distributed as dist
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        tok, rr = _tokens(rank)
        experts = _OracleExperts()
        seen = {}

        def compute(recv_x, recv_local):
            seen["x"] = recv_x.view(torch.int16).numpy().view(np.uint16).copy()
            seen["local"] = recv_local.numpy().copy()
            return _oracle_compute(rank, world, experts)(recv_x, recv_local)

        L = ep.ExpertParallelMoE(rank, world, compute=compute, combine=_oracle_combine)
        x = torch.from_numpy(tok.x_bits.view(np.int16)).view(torch.bfloat16)
        out = L.forward(x, torch.from_numpy(rr.topk_idx), rr.topk_w, ep.DistExchange())
        ex_x, ex_l = _expected_recv(rank, world)
        ok_rows = np.array_equal(seen["x"], ex_x) and np.array_equal(seen["local"], ex_l)
        err = O.rel_l2(out.numpy(), _expected_layer(tok, rr))
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, ok_rows, err, None))
    except Exception as e:  # pragma: no cover - reported to the parent
        q.put((rank, False, float("inf"), repr(e)))


def test_gloo_two_ranks_exchange():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_gloo_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    for rank, ok_rows, err, exc in sorted(res):
        assert exc is None, f"rank {rank}: {exc}"
        assert ok_rows, f"rank {rank} received the wrong rows"
        assert err <= 1e-12, f"rank {rank}: rel-L2 {err}"


def test_plan_empty_batch_and_one_rank():
    """No tokens: every count is zero and every index array empty.  One rank
    (W = 1) owns all 128 experts: every token is one row whose local ids are
    its expert ids, and the returned rows come back in item order."""
    for W in (2, 8):
        p = ep.plan_dispatch(torch.zeros((0, 8), dtype=torch.int32), W)
        assert p.send_counts.tolist() == [0] * W and p.ret_counts.tolist() == [0] * W
        assert p.send_tok.numel() == 0 and p.send_local.shape == (0, 8)
        assert p.ret_index.numel() == 0
    tok, rr = _tokens(0)
    p = ep.plan_dispatch(torch.from_numpy(rr.topk_idx), 1)
    assert p.send_counts.tolist() == [T_PER_RANK] and p.ret_counts.tolist() == [T_PER_RANK * 8]
    assert p.send_tok.tolist() == list(range(T_PER_RANK))
    np.testing.assert_array_equal(p.send_local.numpy(), rr.topk_idx)
    np.testing.assert_array_equal(p.ret_index.numpy(), np.arange(T_PER_RANK * 8))


def test_in_process_with_a_rank_without_tokens():
    """Two ranks, the second with an empty batch: it still serves the rows
    routed to its experts, and the first rank's layer equals the oracle's."""
    experts = _OracleExperts()
    tok, rr = _tokens(0)
    layers = [ep.ExpertParallelMoE(r, 2, compute=_oracle_compute(r, 2, experts),
                                   combine=_oracle_combine) for r in range(2)]
    xs = [torch.from_numpy(tok.x_bits.view(np.int16)).view(torch.bfloat16),
          torch.zeros((0, ep.HIDDEN), dtype=torch.bfloat16)]
    idxs = [torch.from_numpy(rr.topk_idx), torch.zeros((0, 8), dtype=torch.int32)]
    ws = [rr.topk_w, np.zeros((0, 8), np.float32)]
    outs = ep.forward_in_process(layers, xs, idxs, ws)
    assert O.rel_l2(outs[0].numpy(), _expected_layer(tok, rr)) <= 1e-12
    assert tuple(outs[1].shape) == (0, ep.HIDDEN)
    # rank 1 served exactly the rows of rank 0's tokens with an expert in 64..127
    assert sum(layers[1].recv_counts) == int(((rr.topk_idx // 64) == 1).any(axis=1).sum())
