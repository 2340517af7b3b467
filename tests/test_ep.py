"""Expert parallelism on CPU: the exchange schedule of ``ep.ep_forward`` run by
world-size-2 gloo ranks (and by in-process ranks), with each rank's kernels
stood in for by the CPU oracle and plain numpy index operations written here
from the steps' definitions. Checks who sends which rows, how an expert GPU
orders what it receives, and the recombination order: a token's output bits
must equal the single-GPU layer's (the oracle's forward) whatever G is, and
whichever rank holds the token."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import synth

H, E, K, I = 256, 8, 2, 256


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


class OracleSteps:
    """The steps of one rank on the CPU: routing, permutation, the experts' FFN
    and the combine from the oracle; pack, receive plan and row gather as numpy
    index operations following their definitions in include/moe.h. The rank
    holds the weights of its own experts only."""

    def __init__(self, rank, world, seed=0):
        self.G, self.rank, self.K, self.H = world, rank, K, H
        self.E_loc = E // world
        self.e0 = rank * self.E_loc
        self.gu, self.dn = {}, {}
        for e in range(self.e0, self.e0 + self.E_loc):
            g, d = synth.expert_weights(e, H, I, seed=seed)
            self.gu[e], self.dn[e] = oracle.as_u16(g), oracle.as_u16(d)

    def empty(self, shape, dtype):
        return torch.empty(shape, dtype=dtype)

    def to_host(self, t):
        return t

    def route(self, x, wr, bias):
        _, idx, w = oracle.route(oracle.as_u16(x), wr.numpy(), None if bias is None else bias.numpy(), K)
        return torch.from_numpy(idx), torch.from_numpy(w.astype(np.float32))

    def permute(self, idx):
        counts, offsets, ps, pk, inv = oracle.permute(idx.numpy(), E)
        return tuple(torch.from_numpy(np.ascontiguousarray(a)) for a in (counts, offsets, ps, pk, inv))

    def pack(self, x, w, perm_src, perm_k, offsets):
        n = int(offsets[E])
        ps, pk = perm_src.numpy()[:n], perm_k.numpy()[:n]
        x_send = torch.zeros((x.shape[0] * K, H), dtype=torch.bfloat16)
        w_send = torch.zeros((x.shape[0] * K,), dtype=torch.float32)
        x_send[:n] = x[torch.from_numpy(ps).long()]
        w_send[:n] = w[torch.from_numpy(ps).long(), torch.from_numpy(pk).long()]
        return x_send, w_send

    def recv_plan(self, recv_counts, n_rows):
        c = recv_counts.numpy().reshape(self.G, self.E_loc)
        arrival_start = np.concatenate([[0], np.cumsum(c.reshape(-1))[:-1]]).reshape(self.G, self.E_loc)
        perm = []
        offsets = [0]
        for e in range(self.E_loc):  # local expert, then source, then arrival
            for g in range(self.G):
                perm.extend(range(arrival_start[g, e], arrival_start[g, e] + c[g, e]))
            offsets.append(len(perm))
        perm = np.array(perm, dtype=np.int32)
        assert len(perm) == n_rows
        inv = np.empty_like(perm)
        inv[perm] = np.arange(n_rows, dtype=np.int32)
        return (torch.tensor(offsets, dtype=torch.int32), torch.from_numpy(perm),
                torch.zeros(n_rows, dtype=torch.int32), torch.from_numpy(inv))

    def expert_ffn(self, x_recv, perm, perm_k, offsets, w_recv):
        off = offsets.numpy()
        expert = np.repeat(np.arange(self.E_loc), np.diff(off)) + self.e0  # sorted row -> global expert
        p = perm.numpy()
        if len(p) == 0:
            return torch.empty((0, H), dtype=torch.float32)
        y = oracle.ffn_bf16(oracle.as_u16(x_recv), p, expert.astype(np.int32), w_recv.numpy()[p], self.gu, self.dn, E)
        return torch.from_numpy(y)

    def gather_rows(self, y, idx):
        return y[idx.long()]

    def combine(self, y_pair, inv):
        return torch.from_numpy(oracle.combine(y_pair.numpy(), inv.numpy()).view(np.int16)).view(torch.bfloat16)


def _tokens(rank, T):
    return synth.tokens(T, H, seed=0, first_token=1000 * rank)


def _router(bias_kind):
    wr = synth.router_weight(E, H, seed=0)
    if bias_kind == "skew":  # every token's pairs on experts 0 and 1: all rows go to rank 0, none to rank 1
        b = torch.full((E,), -50.0)
        b[0], b[1] = 20.0, 10.0
        return wr, b
    return wr, None


def _reference(rank, T, bias_kind):
    """The single-GPU layer on this rank's tokens: the oracle's forward."""
    x = _tokens(rank, T)
    wr, b = _router(bias_kind)
    gu, dn = {}, {}
    for e in range(E):
        g, d = synth.expert_weights(e, H, I, seed=0)
        gu[e], dn[e] = oracle.as_u16(g), oracle.as_u16(d)
    return oracle.forward(oracle.as_u16(x), wr.numpy(), None if b is None else b.numpy(), K, E, gu, dn)["out"]


def _worker(rank, world, port, q, T_of, bias_kind):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from mixture_experts_layer_24_b200 import ep
    try:
        steps = OracleSteps(rank, world)
        comm = ep.TorchComm()
        wr, b = _router(bias_kind)
        out = ep.ep_forward(steps, comm, _tokens(rank, T_of[rank]), wr, b)
        q.put((rank, oracle.as_u16(out)))
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.parametrize("T_of,bias_kind", [((5, 3), None), ((1, 7), None), ((4, 4), "skew"), ((0, 6), None)])
def test_two_gloo_ranks_match_the_single_gpu_layer(T_of, bias_kind):
    """Two ranks with their own tokens (uneven counts, a rank with no tokens,
    every pair on one rank's experts): each rank's output bits equal the
    single-GPU layer's for its tokens."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, T_of, bias_kind)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        if T_of[r] == 0:
            assert res[r].shape == (0, H)
            continue
        assert np.array_equal(res[r], _reference(r, T_of[r], bias_kind)), f"rank {r}"


@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_output_bits_do_not_depend_on_G(world):
    """The same tokens split over G in-process ranks (threads), G = 1, 2, 4, 8:
    every token's output equals the single-GPU layer's."""
    import threading

    from mixture_experts_layer_24_b200 import ep
    comms = ep.LocalComm.group(world)
    T_of = [3 + r for r in range(world)]
    outs, errs = {}, []

    def run(r):
        try:
            wr, b = _router(None)
            outs[r] = oracle.as_u16(ep.ep_forward(OracleSteps(r, world), comms[r], _tokens(r, T_of[r]), wr, b))
        except Exception as exc:  # surfaced below
            errs.append(exc)
            comms[r].shared.barrier.abort()

    th = [threading.Thread(target=run, args=(r,)) for r in range(world)]
    for t in th:
        t.start()
    for t in th:
        t.join(timeout=300)
    assert not errs, errs
    for r in range(world):
        assert np.array_equal(outs[r], _reference(r, T_of[r], None)), f"rank {r} of {world}"


def test_receive_plan_orders_by_expert_then_source():
    """A hand-built receive: 2 sources x 3 local experts, counts
    [[2, 0, 1], [1, 3, 0]] -> arrival blocks (g0e0: rows 0-1, g0e2: 2,
    g1e0: 3, g1e1: 4-6); sorted by expert then source: 0, 1, 3 | 4, 5, 6 | 2."""
    st = OracleSteps.__new__(OracleSteps)
    st.G, st.E_loc = 2, 3
    off, perm, pk, inv = st.recv_plan(torch.tensor([2, 0, 1, 1, 3, 0], dtype=torch.int32), 7)
    assert off.tolist() == [0, 3, 6, 7]
    assert perm.tolist() == [0, 1, 3, 4, 5, 6, 2]
    assert inv.tolist() == [0, 1, 6, 2, 3, 4, 5]
    assert pk.tolist() == [0] * 7
