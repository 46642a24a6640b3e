"""Expert-parallel routed-MoE layer over a torch.distributed process group.

Rank r of a group of G holds experts [r E/G, (r + 1) E/G) of the layer; the router weights
are on every rank, and every rank keeps its own tokens. A forward of T tokens on a rank:

  1. selection: ids [T, k], w [T, k] for its tokens (libmoe moe_route);
  2. dispatch: the T k slots sorted stably by the rank that holds their expert; one all-to-all
     of the counts, then one of the token rows (bf16 x of each slot, gathered by
     moe_gather_rows) with each slot's local expert id and weight;
  3. experts: the rows this rank received, each through its expert with its weight
     (moe_experts_forward): w s_e FFN_e(x);
  4. return: one all-to-all back of those weighted rows, put back in slot order
     (moe_gather_rows with the inverse order);
  5. combine: out[t] = sum over j of the slot rows, in j order (moe_combine_slots).

This module is host logic only -- plan, collectives and argument marshalling; every step of
the layer itself runs in libmoe's kernels (or, for tests on CPU ranks, in the ops object the
caller passes). The all-to-alls go through torch.distributed (NCCL between GPUs); no TMA and
no cluster multicast is involved. The plan needs the per-destination counts on the host
(they size the exchanges), so a forward synchronises its stream once after the selection.
"""
from __future__ import annotations

import numpy as np


def dispatch_plan(ids: np.ndarray, E: int, world: int):
    """Slots in dispatch order and the rows each rank receives from this one.

    ids: int [T, k] expert ids of this rank's tokens. Returns (order, dest, send_counts):
    order [T k] int32, the slot indices s = t k + j sorted stably by destination rank (so a
    destination receives its rows in slot order); dest [T k] the destination of each slot in
    that order; send_counts [world] int64.
    """
    if E % world:
        raise ValueError(f"E = {E} experts do not split evenly over {world} ranks")
    e_local = E // world
    flat = np.asarray(ids, dtype=np.int64).reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert id outside [0, E)")
    dest_of_slot = flat // e_local
    order = np.argsort(dest_of_slot, kind="stable").astype(np.int32)
    counts = np.bincount(dest_of_slot, minlength=world).astype(np.int64)
    return order, dest_of_slot[order], counts


def inverse_order(order: np.ndarray) -> np.ndarray:
    """inv with inv[order[i]] = i: row i of the returned rows belongs to slot order[i]."""
    inv = np.empty_like(order)
    inv[order] = np.arange(order.size, dtype=order.dtype)
    return inv


class LibmoeOps:
    """The layer's steps on a CUDA device through libmoe (moe_init must have run on it)."""

    def __init__(self, device):
        import torch
        import mixture_experts_gemv_b200 as moe
        self.torch, self.moe, self.device = torch, moe, device

    def tensor(self, a, dtype=None):
        t = self.torch.as_tensor(a, dtype=dtype)
        return t.to(self.device)

    def route(self, x, router_w, router_scale, T, d, E, k):
        torch = self.torch
        ids = torch.empty((T, k), dtype=torch.int32, device=self.device)
        w = torch.empty((T, k), dtype=torch.float32, device=self.device)
        self.moe.moe_route(x, router_w, router_scale, T, d, E, k, ids, w)
        return ids, w

    def gather(self, src, index, n, row_elems):
        torch = self.torch
        dst = torch.empty((n, row_elems), dtype=src.dtype, device=self.device)
        if n:
            self.moe.moe_gather_rows(src, index, n, row_elems * src.element_size(), dst)
        return dst

    def experts(self, x_rows, e_rows, w_rows, gate_up, down, expert_scale, R, d, f, e_local):
        torch = self.torch
        out = torch.empty((R, d), dtype=torch.float32, device=self.device)
        if R:
            self.moe.moe_experts_forward(x_rows, e_rows, w_rows, gate_up, down, expert_scale, R, d, f, e_local, out)
        return out

    def combine(self, y_slots, T, d, k):
        torch = self.torch
        out = torch.empty((T, d), dtype=torch.float32, device=self.device)
        if T:
            self.moe.moe_combine_slots(y_slots, T, d, k, out)
        return out

    def to_host(self, t):
        self.torch.cuda.current_stream(self.device).synchronize()
        return t.cpu().numpy()


class ExpertParallelLayer:
    """One routed-MoE layer whose experts are split evenly over the ranks of `group`."""

    def __init__(self, E: int, d: int, f: int, k: int, ops, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if E % self.world:
            raise ValueError(f"E = {E} experts do not split evenly over {self.world} ranks")
        self.E, self.d, self.f, self.k = E, d, f, k
        self.e_local = E // self.world
        self.expert_base = self.rank * self.e_local
        self.ops = ops

    def _exchange(self, send, send_counts, recv_counts, row_shape, dtype):
        import torch
        recv = torch.empty((int(recv_counts.sum()),) + tuple(row_shape), dtype=dtype, device=send.device)
        self.dist.all_to_all_single(recv, send, [int(c) for c in recv_counts], [int(c) for c in send_counts],
                                    group=self.group)
        return recv

    def forward(self, x, router_w, router_scale, gate_up_local, down_local, expert_scale_local, T: int):
        """x: this rank's tokens, bf16 bits [T, d] (int16 tensor); the local experts' weights.
        Returns out fp32 [T, d] for this rank's tokens."""
        import torch
        ops, d, k = self.ops, self.d, self.k
        ids, w = ops.route(x, router_w, router_scale, T, d, self.E, k)
        ids_h, w_h = ops.to_host(ids), ops.to_host(w)
        order, dest, send_counts = dispatch_plan(ids_h, self.E, self.world)
        counts_t = ops.tensor(send_counts, dtype=torch.int64)
        recv_counts_t = torch.empty_like(counts_t)
        self.dist.all_to_all_single(recv_counts_t, counts_t, group=self.group)
        recv_counts = ops.to_host(recv_counts_t).astype(np.int64)
        S = T * k
        # rows out, in dispatch order: the slot's token row, local expert id and weight
        tok = ops.tensor((order // k).astype(np.int32), dtype=torch.int32)
        x_send = ops.gather(x, tok, S, d)
        e_send = ops.tensor((ids_h.reshape(-1)[order] - dest * self.e_local).astype(np.int32), dtype=torch.int32)
        w_send = ops.tensor(w_h.reshape(-1)[order], dtype=w.dtype)
        # bf16 rows travel as their bytes (the collectives have no 16-bit integer type)
        x_recv = self._exchange(x_send.view(torch.uint8), send_counts, recv_counts, (2 * d,), torch.uint8)
        x_recv = x_recv.view(x.dtype)
        e_recv = self._exchange(e_send, send_counts, recv_counts, (), torch.int32)
        w_recv = self._exchange(w_send, send_counts, recv_counts, (), w.dtype)
        R = int(recv_counts.sum())
        y_recv = ops.experts(x_recv, e_recv, w_recv, gate_up_local, down_local, expert_scale_local, R, d, self.f,
                             self.e_local)
        y_back = self._exchange(y_recv, recv_counts, send_counts, (d,), y_recv.dtype)
        y_slots = ops.gather(y_back, ops.tensor(inverse_order(order), dtype=torch.int32), S, d)
        return ops.combine(y_slots, T, d, k)
