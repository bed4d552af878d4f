"""Expert parallelism over G ranks, one process per GPU.

Rank r holds the experts [r * E / G, (r + 1) * E / G) of the layer as a
PackedLayer of E / G experts. A forward call on a rank's tokens:

1. routes every slot to the rank that holds its expert (e4b_ep_dest, then the
   routing pass with E = G ranks), and packs the routed rows in that order
   with their local expert ids and gates (e4b_ep_pack);
2. exchanges the per-rank row counts, then the rows, ids and gates, with
   all-to-all collectives (NCCL over NVLink; the split sizes need the counts
   on the host, one small device-to-host copy a call);
3. runs the rank's experts on the rows it received, one slot a row, gate
   applied (e4b_moe_forward with top_k = 1);
4. sends the outputs back with the reverse all-to-all and sums each token's
   rows (e4b_ep_combine).

The pages describe a one-GPU layer; this split is the library's own. Each
slot's output is rounded to bf16 before the sum, so y differs from the
one-GPU layer by at most top_k bf16 roundings. The device work is done by the
`ops` object (the library's kernels by default); tests on CPU ranks pass an
object with the same methods.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import e4b


class CudaOps:
    """The library's kernels for the device steps of an expert-parallel call."""

    def dest(self, ids, E, epr):
        dest = torch.empty_like(ids)
        e4b.e4b_ep_dest(ids, E, epr, dest)
        return dest

    def route(self, dest, G):
        counts, offsets, perm, inv, _ = e4b.route(dest, G)
        return counts, offsets, perm, inv

    def pack(self, x, ids, gates, perm, offsets, G, R, epr):
        n = max(R, 1)
        xs = torch.empty((n, x.shape[1]), dtype=x.dtype, device=x.device)
        lids = torch.empty(n, dtype=torch.int32, device=x.device)
        gs = torch.empty(n, dtype=torch.float32, device=x.device)
        e4b.e4b_ep_pack(x, ids, gates, perm, offsets, G, R, epr, xs, lids, gs)
        return xs[:R], lids[:R], gs[:R]

    def local_forward(self, layer, x_in, lids, gates):
        if x_in.shape[0] == 0:
            return torch.empty_like(x_in)
        return e4b.moe_forward(layer, x_in, lids.reshape(-1, 1).contiguous(), gates.reshape(-1, 1).contiguous())

    def combine(self, ys, inv, T, k, H, like):
        y = torch.empty((T, H), dtype=like.dtype, device=like.device)
        if ys.shape[0] == 0:
            ys = torch.zeros((1, H), dtype=like.dtype, device=like.device)
        e4b.e4b_ep_combine(ys, inv, T, k, y)
        return y


class ExpertParallelLayer:
    """The layer split over the ranks of `group`: `local` holds this rank's
    E / G experts of the E-expert layer."""

    def __init__(self, local, E: int, group=None, ops=None):
        self.G = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if E % self.G or local.E != E // self.G:
            raise ValueError(f"{E} experts over {self.G} ranks: each rank holds {E // self.G}, got {local.E}")
        self.local, self.E, self.group = local, E, group
        self.epr = E // self.G
        self.ops = ops or CudaOps()

    def _exchange(self, send, send_splits, recv_splits, rows_shape):
        out = torch.empty(rows_shape, dtype=send.dtype, device=send.device)
        dist.all_to_all_single(out, send.contiguous(), recv_splits, send_splits, group=self.group)
        return out

    def forward(self, x, ids, gates):
        """y [T, H] for this rank's tokens x [T, H] with global expert ids and
        gates [T, k]."""
        T, k = ids.shape
        H = x.shape[1]
        o = self.ops
        dest = o.dest(ids, self.E, self.epr)
        counts, offsets, perm, inv = o.route(dest, self.G)
        recv_counts = torch.empty_like(counts)
        dist.all_to_all_single(recv_counts, counts, group=self.group)
        send_splits = [int(c) for c in counts.cpu()]
        recv_splits = [int(c) for c in recv_counts.cpu()]
        R, R_in = sum(send_splits), sum(recv_splits)
        xs, lids, gs = o.pack(x, ids, gates, perm, offsets, self.G, R, self.epr)
        x_in = self._exchange(xs, send_splits, recv_splits, (R_in, H))
        lid_in = self._exchange(lids, send_splits, recv_splits, (R_in,))
        g_in = self._exchange(gs, send_splits, recv_splits, (R_in,))
        y_in = o.local_forward(self.local, x_in, lid_in, g_in)
        ys = self._exchange(y_in, recv_splits, send_splits, (R, H))
        return o.combine(ys, inv, T, k, H, x)
