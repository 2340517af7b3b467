"""Expert parallelism: the routed MoE layer over G GPUs, experts split by range.

GPU g holds experts [g*E/G, (g+1)*E/G) and its own tokens. One forward:

1. token GPU: route and permute its tokens over all E experts (libmoe); the
   sorted pairs are grouped by expert, hence by the GPU that holds the expert;
   ``moe_ep_pack`` lays the x rows and routing weights out in that order;
2. exchange: an all-to-all of the per-expert counts, then of the rows and
   weights (NCCL through ``torch.distributed``; the split sizes come from the
   counts, read on the host once);
3. expert GPU: ``moe_ep_recv_plan`` orders the received rows by local expert,
   ``moe_expert_ffn`` computes them (a context with E/G experts and top-1:
   each received row is one pair, its routing weight applied in the down
   epilogue), ``moe_ep_gather_rows`` puts the results back in arrival order;
4. exchange back: the reverse all-to-all returns every y_pair row to its
   token's GPU, in that GPU's sorted order;
5. token GPU: ``moe_combine`` sums each token's pairs in k order.

The pages split each expert across their GPUs and sum the slices over NCCL
(vLLM-Moet, topairepos.com page, hybrid results table, row "the step"; model
table, "one expert as its 576-row slices"). That sum would change the order of
a token's additions across GPUs; here whole pairs move, each pair's result is
the same fp32 value whatever rows share its tile, and the combine runs on the
token's GPU in k order, so a token's output bits do not depend on G.

Every step of the arithmetic runs in libmoe's kernels. This module is the
schedule: which call comes when, the split sizes, and the collectives. The
steps are an object (``LibmoeSteps``) so that the same schedule can be driven
by another implementation of them.
"""

from __future__ import annotations

import threading

import torch

from .binding import (MOE_BF16, MOE_LOC_HBM, MoeLayer, check_tensor, moe_ep_gather_rows, moe_ep_pack,
                      moe_ep_recv_plan)


class TorchComm:
    """all-to-all over a torch.distributed process group (NCCL on GPUs)."""

    def __init__(self, group=None):
        self.group = group
        self.rank = torch.distributed.get_rank(group)
        self.world = torch.distributed.get_world_size(group)

    def all_to_all(self, out, inp, out_splits, in_splits):
        torch.distributed.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)


class LocalComm:
    """all-to-all among G ranks that are threads of one process (each rank's
    kernels on its own stream; nothing on the device waits for another rank:
    the host moves the rows between the ranks' buffers after a barrier)."""

    class _Shared:
        def __init__(self, world):
            self.world = world
            self.barrier = threading.Barrier(world)
            self.slots = [None] * world

    def __init__(self, shared, rank):
        self.shared, self.rank, self.world = shared, rank, shared.world

    @classmethod
    def group(cls, world):
        sh = cls._Shared(world)
        return [cls(sh, r) for r in range(world)]

    def all_to_all(self, out, inp, out_splits, in_splits):
        sh = self.shared
        if inp.is_cuda:
            torch.cuda.current_stream().synchronize()  # this rank's input is complete before others read it
        sh.slots[self.rank] = (inp, list(in_splits))
        sh.barrier.wait()
        at = 0
        for src in range(self.world):
            s_inp, s_splits = sh.slots[src]
            start = sum(s_splits[:self.rank])
            n = s_splits[self.rank]
            assert n == out_splits[src], "split sizes disagree between ranks"
            out[at:at + n].copy_(s_inp[start:start + n])
            at += n
        if out.is_cuda:
            torch.cuda.current_stream().synchronize()
        sh.barrier.wait()  # every rank has copied out of every other rank's input


class LibmoeSteps:
    """The steps of one rank, as libmoe calls: a context over all E experts
    (routing, permutation, pack, combine) and one over this rank's experts
    with top-1 (the received pairs)."""

    def __init__(self, hidden, n_experts, top_k, intermediate, rank, world, wdtype=MOE_BF16, device=None,
                 flags=0):
        if n_experts % world:
            raise ValueError(f"{n_experts} experts do not split evenly over {world} GPUs")
        self.H, self.E, self.K, self.I = hidden, n_experts, top_k, intermediate
        self.G, self.rank = world, rank
        self.E_loc = n_experts // world
        self.e0 = rank * self.E_loc
        self.router = MoeLayer(hidden, n_experts, top_k, intermediate, wdtype, device=device, flags=flags)
        self.local = MoeLayer(hidden, self.E_loc, 1, intermediate, wdtype, device=self.router.device, flags=flags)
        self.device = self.router.device

    # ---- allocation and host reads
    def empty(self, shape, dtype):
        return torch.empty(shape, dtype=dtype, device=self.device)

    def to_host(self, t):
        return t.cpu()

    # ---- experts of this rank (global ids)
    def register(self, e, w_gu, w_dn, s_gu=None, s_dn=None, location=MOE_LOC_HBM):
        if not self.e0 <= e < self.e0 + self.E_loc:
            raise ValueError(f"expert {e} is not held by rank {self.rank} (experts {self.e0}..{self.e0 + self.E_loc - 1})")
        self.local.register(e - self.e0, w_gu, w_dn, s_gu, s_dn, location)

    # ---- the kernels
    def route(self, x, wr, bias):
        return self.router.route(x, wr, bias)

    def permute(self, idx):
        return self.router.permute(idx)

    def pack(self, x, w, perm_src, perm_k, offsets):
        T = x.shape[0]
        x_send = self.empty((T * self.K, self.H), torch.bfloat16)
        w_send = self.empty((T * self.K,), torch.float32)
        moe_ep_pack(self.router.ctx, x, w, perm_src, perm_k, offsets, T, x_send, w_send)
        return x_send, w_send

    def recv_plan(self, recv_counts, n_rows):
        check_tensor(recv_counts, "recv_counts", torch.int32, (self.G * self.E_loc,), self.device)
        offsets = self.empty((self.E_loc + 1,), torch.int32)
        perm = self.empty((n_rows,), torch.int32)
        perm_k = self.empty((n_rows,), torch.int32)
        inv = self.empty((n_rows,), torch.int32)
        moe_ep_recv_plan(self.local.ctx, recv_counts, self.G, offsets, perm, perm_k, inv)
        return offsets, perm, perm_k, inv

    def expert_ffn(self, x_recv, perm, perm_k, offsets, w_recv):
        return self.local.expert_ffn(x_recv, perm, perm_k, offsets, w_recv.view(-1, 1))

    def gather_rows(self, y, idx):
        n = idx.shape[0]
        out = self.empty((n, self.H), torch.float32)
        moe_ep_gather_rows(self.local.ctx, y, idx, n, out)
        return out

    def combine(self, y_pair, inv):
        return self.router.combine(y_pair, inv)

    def status(self):
        return self.router.status() | self.local.status()

    def close(self):
        self.router.close()
        self.local.close()


def ep_forward(steps, comm, x, w_router, logit_bias=None):
    """One expert-parallel forward of this rank's tokens x [T, H]; returns
    out [T, H]. Every rank calls it at the same time (it runs three
    all-to-alls and reads the per-expert counts on the host once)."""
    G, E_loc, K, H = steps.G, steps.E_loc, steps.K, steps.H
    T = x.shape[0]
    idx, w = steps.route(x, w_router, logit_bias)
    counts, offsets, perm_src, perm_k, inv = steps.permute(idx)
    x_send, w_send = steps.pack(x, w, perm_src, perm_k, offsets)
    # counts: rank r sends counts[g*E_loc:(g+1)*E_loc] to g and receives, from each
    # source, the counts of its own experts in the source's sorted order
    recv_counts = steps.empty((G * E_loc,), torch.int32)
    comm.all_to_all(recv_counts, counts, [E_loc] * G, [E_loc] * G)
    c_host = steps.to_host(counts).reshape(G, E_loc).sum(1)
    r_host = steps.to_host(recv_counts).reshape(G, E_loc).sum(1)
    send_splits = [int(v) for v in c_host]
    recv_splits = [int(v) for v in r_host]
    P_valid, R = sum(send_splits), sum(recv_splits)
    x_recv = steps.empty((R, H), torch.bfloat16)
    w_recv = steps.empty((R,), torch.float32)
    comm.all_to_all(x_recv, x_send[:P_valid], recv_splits, send_splits)
    comm.all_to_all(w_recv, w_send[:P_valid], recv_splits, send_splits)
    offsets_loc, perm_loc, pk_loc, inv_loc = steps.recv_plan(recv_counts, R)
    y_loc = steps.expert_ffn(x_recv, perm_loc, pk_loc, offsets_loc, w_recv)
    y_back = steps.gather_rows(y_loc, inv_loc)
    y_pair = steps.empty((T * K, H), torch.float32)
    comm.all_to_all(y_pair[:P_valid], y_back, send_splits, recv_splits)
    return steps.combine(y_pair, inv)
