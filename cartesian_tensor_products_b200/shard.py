"""One graph spread over several GPUs by contiguous receiver ranges.

The edge convolution (FlashCart Sec. 4 Eq. 1) sums, for every receiver, over
that receiver's own incoming edges, so a receiver-sorted graph cuts into
contiguous receiver ranges whose outputs are disjoint: each rank holds its
range's edges, their weights and edge vectors, and the features of the nodes
it owns (the same range).  The data-path exchanges are the ones the sums
force:

  forward   every rank needs the features of all senders: one all-gather of
            the owned feature rows;
  VJP       the sender gradient x_bar collects contributions from every
            range: one reduce-scatter of the per-range partial sums back to
            the owners; w_bar and r_bar are per edge and stay local;
  ladder    node-local (Sec. 5 Eq. 2): each rank runs its own nodes, and only
            the weight gradients (path weights, mixing matrices) are summed
            over ranks with one all-reduce.

This module holds the partition and those collectives (torch.distributed,
NCCL on GPUs, gloo on CPU).  The per-range compute is passed in as a
function, so the same plumbing drives the library's kernels on the GPU
(edge_conv_fn / edge_conv_vjp_fn below, through fc_edge_conv_rect and
fc_edge_conv_vjp_rect) and any other implementation of the same call.
Feature rows are padded to the largest range so that every rank moves
equal-sized blocks.
"""
import numpy as np
import torch
import torch.distributed as dist


def receiver_ranges(rowptr, world):
    """Bounds b[0] = 0 <= b[1] <= ... <= b[world] = N of contiguous receiver
    ranges with near-equal edge counts (rank r owns [b[r], b[r+1]))."""
    rowptr = np.asarray(rowptr, dtype=np.int64)
    N = len(rowptr) - 1
    E = int(rowptr[-1])
    bounds = [0]
    for r in range(1, world):
        if E > 0:
            u = int(np.searchsorted(rowptr, E * r / world, side="left"))
        else:
            u = (N * r) // world
        bounds.append(min(max(u, bounds[-1]), N))
    bounds.append(N)
    return bounds


def rowptr_of(receivers, n_nodes):
    """Row pointer [n_nodes+1] of receiver-sorted receiver indices."""
    return np.searchsorted(np.asarray(receivers), np.arange(n_nodes + 1), side="left")


class GraphShard:
    """Rank `rank`'s part of a receiver-sorted graph: receivers
    [u0, u1) renumbered from 0, senders kept global, edges [e0, e1)."""

    def __init__(self, edge_index, n_nodes, rank, world, bounds=None):
        edge_index = np.asarray(edge_index)
        rp = rowptr_of(edge_index[0], n_nodes)
        self.bounds = receiver_ranges(rp, world) if bounds is None else list(bounds)
        self.rank, self.world, self.n_nodes = rank, world, n_nodes
        self.u0, self.u1 = self.bounds[rank], self.bounds[rank + 1]
        self.e0, self.e1 = int(rp[self.u0]), int(rp[self.u1])
        self.n_local = self.u1 - self.u0
        self.nmax = max(self.bounds[i + 1] - self.bounds[i] for i in range(world))
        ei = edge_index[:, self.e0:self.e1].astype(np.int32)
        self.edge_index = np.stack([ei[0] - self.u0, ei[1]]).astype(np.int32)

    def local_edges(self, per_edge):
        """Rows [e0, e1) of a per-edge array (weights, edge vectors)."""
        return per_edge[self.e0:self.e1]

    def local_nodes(self, per_node):
        """Rows [u0, u1) of a per-node array."""
        return per_node[self.u0:self.u1]

    def _pad(self, rows):
        out = rows.new_zeros((self.nmax,) + tuple(rows.shape[1:]))
        out[:rows.shape[0]] = rows
        return out

    def equal_ranges(self):
        return all(self.bounds[r + 1] - self.bounds[r] == self.nmax for r in range(self.world))

    def gather_rows(self, local_rows, group=None, out=None):
        """All ranks' owned rows -> the whole graph's [N, ...] (all-gather).
        With equal ranges the blocks land in place (into `out` if given)."""
        assert local_rows.shape[0] == self.n_local
        shape = (self.world * self.nmax,) + tuple(local_rows.shape[1:])
        if self.equal_ranges():
            blocks = out if out is not None else torch.empty(shape, dtype=local_rows.dtype,
                                                             device=local_rows.device)
            dist.all_gather_into_tensor(blocks, local_rows.contiguous(), group=group)
            return blocks
        blocks = torch.empty(shape, dtype=local_rows.dtype, device=local_rows.device)
        dist.all_gather_into_tensor(blocks, self._pad(local_rows).contiguous(), group=group)
        parts = [blocks[r * self.nmax:r * self.nmax + self.bounds[r + 1] - self.bounds[r]]
                 for r in range(self.world)]
        return torch.cat(parts, 0)

    def reduce_scatter_rows(self, full_partial, group=None):
        """Per-rank partial sums over all N rows -> this rank's owned rows of
        their sum over ranks (reduce-scatter)."""
        assert full_partial.shape[0] == self.n_nodes
        blocks = full_partial.new_zeros((self.world * self.nmax,) + tuple(full_partial.shape[1:]))
        for r in range(self.world):
            a, b = self.bounds[r], self.bounds[r + 1]
            blocks[r * self.nmax:r * self.nmax + b - a] = full_partial[a:b]
        out = full_partial.new_empty((self.nmax,) + tuple(full_partial.shape[1:]))
        dist.reduce_scatter_tensor(out, blocks, op=dist.ReduceOp.SUM, group=group)
        return out[:self.n_local]


def conv_forward(shard, conv_fn, x_local, edge_vec_local, w_local, group=None):
    """z rows of this rank's receivers: gather every sender's features, then
    conv_fn(edge_index_local, edge_vec_local, x_all, w_local, n_local) over
    the local edges (receivers local, senders global)."""
    x_all = shard.gather_rows(x_local, group)
    return conv_fn(shard.edge_index, edge_vec_local, x_all, w_local, shard.n_local)


def conv_vjp(shard, vjp_fn, x_local, edge_vec_local, w_local, g_local, group=None):
    """(x_bar of the owned nodes, w_bar and r_bar of the local edges):
    vjp_fn(edge_index_local, edge_vec_local, x_all, w_local, g_local,
    n_local) returns the range's partial x_bar over all N senders, which one
    reduce-scatter sums into the owners' rows."""
    x_all = shard.gather_rows(x_local, group)
    xb_partial, wb, rb = vjp_fn(shard.edge_index, edge_vec_local, x_all, w_local, g_local,
                                shard.n_local)
    return shard.reduce_scatter_rows(xb_partial, group), wb, rb


def ladder_vjp(node_shard, ladder_vjp_fn, A1_local, gz_local, group=None):
    """Node-partitioned ladder VJP: ladder_vjp_fn(A1_local, gz_local) returns
    (A1_bar_local, path_w_bar, mix_w_bar) over the local nodes; the weight
    gradients are summed over ranks (all-reduce)."""
    a1b, pwb, mwb = ladder_vjp_fn(A1_local, gz_local)
    if pwb is not None and pwb.numel():
        dist.all_reduce(pwb, op=dist.ReduceOp.SUM, group=group)
    if mwb is not None and mwb.numel():
        dist.all_reduce(mwb, op=dist.ReduceOp.SUM, group=group)
    return a1b, pwb, mwb


def edge_conv_fn(lmax, sum_paths=False):
    """conv_fn for conv_forward on the library's kernels (fc_edge_conv_rect)."""
    from cartesian_tensor_products_b200 import flashcart as fc

    def f(edge_index, edge_vec, x_all, w, n_local):
        ei = torch.as_tensor(edge_index, device=x_all.device)
        rp = fc.build_rowptr(ei, edge_vec, n_local, n_send=x_all.shape[0])
        return fc.edge_conv(lmax, rp, ei, edge_vec, x_all, w, sum_paths=sum_paths)
    return f


def edge_conv_vjp_fn(lmax, sum_paths=False):
    """vjp_fn for conv_vjp on the library's kernels (fc_edge_conv_vjp_rect)."""
    from cartesian_tensor_products_b200 import flashcart as fc

    def f(edge_index, edge_vec, x_all, w, g, n_local):
        ei = torch.as_tensor(edge_index, device=x_all.device)
        rp = fc.build_rowptr(ei, edge_vec, n_local, n_send=x_all.shape[0])
        return fc.edge_conv_vjp(lmax, rp, ei, edge_vec, x_all, w, g, sum_paths=sum_paths)
    return f
