"""Table-wise model parallelism of the embedding tables with data-parallel MLPs.

The system the pages describe keeps the embedding tables model-parallel and
the fully connected layers data-parallel, with an all-to-all of the embedding
lookup results in between (arXiv 1906.00091 index page, Abstract;
science.uptrusthq.com citation snippet on all-to-all communication of the
lookups; "DLRM", briansu.co, section 5). Here:

  * each rank owns a contiguous range of tables (ShardPlan: the split that
    minimises the largest rank's table bytes) and holds only their rows;
  * a global batch of B = world x B_local samples: rank r has the dense
    features and labels of its shard (samples r B_local .. (r+1) B_local - 1)
    and the bags of its own tables for all B samples (shard_bags cuts them
    out of the table-major CSR);
  * forward: the rank pools its own tables' bags for all B samples
    (dlrm_embbag_fwd), one all-to-all sends every rank the rows of its shard,
    dlrm_pooled_assemble places them, and the bottom MLP, the interaction and
    the top MLP run on the rank's shard (dlrm_mlp_fwd, dlrm_interact_fwd);
  * training: dlrm_backward_pooled gives the shard's MLP gradients and the
    gradient of every pooled vector; dlrm_pooled_split cuts the latter per
    owner and the reverse all-to-all brings each owner its tables' gradients
    for all B samples, which dlrm_embbag_sgd applies (row-sorted, in
    occurrence order); the MLP gradients are summed by one all-reduce and
    applied by dlrm_mlp_sgd. Every rank computes the mean loss of its shard,
    so both updates take lr / world: the step is plain SGD on the mean loss
    of the global batch.

Every arithmetic step runs in libdlrm's kernels; this module only decides
what goes where and calls torch.distributed for the two exchanges (NCCL over
NVLink between GPUs, gloo between CPU processes). The pooled vectors cross
as fp32. No collective is issued on another stream than the caller's, and
every rank issues the same collectives in the same order.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch
import torch.distributed as dist

from . import _abi as E


@dataclass(frozen=True)
class ShardPlan:
    """Rank r owns tables first[r] .. first[r] + count[r] - 1 (contiguous, in table order)."""
    world: int
    first: tuple
    count: tuple

    @property
    def K(self) -> int:
        return self.first[-1] + self.count[-1]

    def owner(self, k: int) -> int:
        for r in range(self.world):
            if self.first[r] <= k < self.first[r] + self.count[r]:
                return r
        raise IndexError(k)

    def tables_of(self, r: int) -> range:
        return range(self.first[r], self.first[r] + self.count[r])


def plan_tables(table_bytes, world: int) -> ShardPlan:
    """Contiguous ranges of tables, one per rank, that minimise the largest rank's bytes (exact dynamic
    programme over split points; ties go to the earliest split). Ranks may own no table when there are
    fewer tables than ranks."""
    sizes = [int(x) for x in table_bytes]
    K = len(sizes)
    if world < 1 or K < 1:
        raise ValueError("need at least one table and one rank")
    pre = np.concatenate([[0], np.cumsum(sizes, dtype=np.int64)])
    INF = np.iinfo(np.int64).max
    # best[r][k]: smallest largest-part over splits of tables 0..k-1 into r parts; cut[r][k]: start of the last
    best = np.full((world + 1, K + 1), INF, dtype=np.int64)
    cut = np.zeros((world + 1, K + 1), dtype=np.int64)
    best[0][0] = 0
    for r in range(1, world + 1):
        for k in range(K + 1):
            for j in range(k + 1):           # the r-th part is tables j .. k-1 (possibly empty)
                if best[r - 1][j] == INF:
                    continue
                v = max(int(best[r - 1][j]), int(pre[k] - pre[j]))
                if v < best[r][k]:
                    best[r][k], cut[r][k] = v, j
    starts = []
    k = K
    for r in range(world, 0, -1):
        j = int(cut[r][k])
        starts.append((j, k - j))
        k = j
    starts.reverse()
    return ShardPlan(world, tuple(s for s, _ in starts), tuple(c for _, c in starts))


def shard_bags(offsets, indices, B: int, first: int, count: int):
    """The CSR of tables first .. first + count - 1 for all B samples, cut out of a table-major CSR
    (offsets [K B + 1]) and rebased to start at 0. Returns (offsets [count B + 1], indices)."""
    offs = np.asarray(offsets, np.int64)
    lo, hi = int(offs[first * B]), int(offs[(first + count) * B])
    own = (offs[first * B:(first + count) * B + 1] - lo).astype(np.int32)
    return own, np.asarray(indices)[lo:hi]


def split_sizes(plan: ShardPlan, rank: int, B_local: int, d: int):
    """Element counts of the forward all-to-all on `rank`: it sends B_local x count[rank] x d to every rank
    and receives B_local x count[s] x d from every rank s."""
    send = [B_local * plan.count[rank] * d] * plan.world
    recv = [B_local * plan.count[s] * d for s in range(plan.world)]
    return send, recv


def exchange_pooled(pooled_own: torch.Tensor, plan: ShardPlan, rank: int, group=None) -> list:
    """pooled_own: [B][count[rank]][d] fp32 (this rank's tables, whole batch, sample-major, so the rows of
    every shard are contiguous). Returns the parts of this rank's shard: parts[s] = [B_local][count[s]][d]."""
    B, _, d = pooled_own.shape
    B_local = B // plan.world
    send, recv = split_sizes(plan, rank, B_local, d)
    out = torch.empty(sum(recv), dtype=pooled_own.dtype, device=pooled_own.device)
    dist.all_to_all_single(out, pooled_own.reshape(-1), output_split_sizes=recv, input_split_sizes=send, group=group)
    parts, o = [], 0
    for s in range(plan.world):
        parts.append(out[o:o + recv[s]].view(B_local, plan.count[s], d))
        o += recv[s]
    return parts


def exchange_grads(parts: list, plan: ShardPlan, rank: int, group=None) -> torch.Tensor:
    """The reverse exchange: parts[s] = [B_local][count[s]][d] gradients of this rank's shard for owner s's
    tables. Returns [B][count[rank]][d]: this rank's tables' gradients for the whole batch, in sample order."""
    B_local, d = parts[0].shape[0], parts[0].shape[2]
    send = [B_local * plan.count[s] * d for s in range(plan.world)]
    recv = [B_local * plan.count[rank] * d] * plan.world
    inp = torch.cat([p.reshape(-1) for p in parts])
    out = torch.empty(sum(recv), dtype=inp.dtype, device=inp.device)
    dist.all_to_all_single(out, inp, output_split_sizes=recv, input_split_sizes=send, group=group)
    return out.view(plan.world * B_local, plan.count[rank], d)


class ShardedDLRM:
    """One rank of a table-wise sharded DLRM on its GPU. tables_own: Tables of this rank's tables only (rows
    first[rank] .. of the global model; None for a rank that owns no table); bot, top: this rank's replicas
    of the MLPs (fp32 for training)."""

    def __init__(self, plan: ShardPlan, rank: int, tables_own, bot, top, d: int, B_local: int, group=None):
        self.plan, self.rank, self.T, self.bot, self.top = plan, rank, tables_own, bot, top
        self.d, self.B_local, self.group = d, B_local, group
        self.B = B_local * plan.world
        K = plan.K
        dev = bot.Ws[0].device
        mlp_dt = E.DT_TORCH[bot.dt]
        self.ld = E.dlrm_ld(d + K * (K + 1) // 2, bot.dt)
        self.pooled_own = torch.empty((self.B, plan.count[rank], d), device=dev)
        self.pooled = torch.empty((B_local, K, d), device=dev)
        self.x_dense = torch.empty((B_local, d), device=dev)
        self.concat = torch.zeros((B_local, self.ld), dtype=mlp_dt, device=dev)
        ws_bytes = max(E.dlrm_mlp_workspace_size(bot, B_local, torch.float32),
                       E.dlrm_mlp_workspace_size(top, B_local, mlp_dt), E.ERR_RECORD_BYTES)
        self.ws = E.alloc_workspace(ws_bytes, dev)
        self.ws_own = E.alloc_workspace(E.ERR_RECORD_BYTES, dev)

    def forward(self, dense_local, offsets_own, indices_own, y_local):
        """y_local [B_local] = sigmoid(top([x_dense, Z])) for this rank's shard."""
        plan, r = self.plan, self.rank
        if plan.count[r]:
            E.dlrm_embbag_fwd(self.T, self.B, offsets_own, indices_own, self.pooled_own, None, self.ws_own)
        parts = exchange_pooled(self.pooled_own, plan, r, self.group)
        E.dlrm_pooled_assemble(self.B_local, plan.K, self.d, plan.first, plan.count, parts, self.pooled)
        E.dlrm_mlp_fwd(self.bot, self.B_local, dense_local, self.bot.dims[0], self.x_dense, self.d, E.ACT_RELU, self.ws)
        E.dlrm_interact_fwd(self.B_local, plan.K, self.d, self.x_dense, self.pooled, self.concat, self.ld)
        E.dlrm_mlp_fwd(self.top, self.B_local, self.concat, self.ld, y_local, 1, E.ACT_SIGMOID, self.ws)
        return y_local

    def _train_buffers(self):
        if getattr(self, "_grads", None) is None:
            K, d, B_l = self.plan.K, self.d, self.B_local
            dev = self.pooled.device
            self._grads = torch.zeros(E.dlrm_grads_pooled_size(K, d, self.bot, self.top, B_l), dtype=torch.uint8,
                                      device=dev)
            self._gofs = E.dlrm_grads_pooled_offsets(K, d, self.bot, self.top, B_l)
            self._tws = E.alloc_workspace(E.dlrm_backward_pooled_workspace_size(K, d, self.bot, self.top, B_l), dev)
            self._dE_parts = [torch.empty((B_l, c, d), device=dev) for c in self.plan.count]
            self._loss = torch.zeros(1, device=dev)
        return self._grads

    def train_step(self, dense_local, offsets_own, indices_own, labels_local, lr: float):
        """One SGD step on the mean loss of the global batch. Returns this rank's shard loss (device scalar)."""
        plan, r, K, d, B_l = self.plan, self.rank, self.plan.K, self.d, self.B_local
        grads = self._train_buffers()
        if plan.count[r]:
            E.dlrm_embbag_fwd(self.T, self.B, offsets_own, indices_own, self.pooled_own, None, self.ws_own)
        parts = exchange_pooled(self.pooled_own, plan, r, self.group)
        E.dlrm_pooled_assemble(B_l, K, d, plan.first, plan.count, parts, self.pooled)
        E.dlrm_backward_pooled(K, d, self.bot, self.top, B_l, dense_local, self.pooled, labels_local, grads,
                               self._tws, loss=self._loss)
        dE = E.grads_view(grads, self._gofs["dE"], (B_l, K, d))
        E.dlrm_pooled_split(B_l, K, d, plan.first, plan.count, dE, self._dE_parts)
        dE_own = exchange_grads(self._dE_parts, plan, r, self.group)
        step = lr / plan.world
        if plan.count[r]:
            scratch = self._sgd_scratch(indices_own.numel())
            E.dlrm_embbag_sgd(self.T, self.B, offsets_own, indices_own, dE_own, step, scratch)
        dense = grads[:self._gofs["dense_end"]].view(torch.float32)
        dist.all_reduce(dense, group=self.group)
        E.dlrm_mlp_sgd(K, d, self.bot, self.top, B_l, step, grads)
        return self._loss

    def _sgd_scratch(self, nnz: int):
        need = E.dlrm_embbag_sgd_scratch_size(self.T, self.B, nnz)
        if getattr(self, "_scratch", None) is None or self._scratch.numel() < need:
            self._scratch = E.alloc_workspace(need, self.pooled.device)
        return self._scratch
