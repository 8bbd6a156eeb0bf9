"""One graph spread over two ranks by receiver range (gloo on CPU, world
size 2), with the FP64 oracle as the per-range compute: the concatenated
convolution outputs (FlashCart Sec. 4 Eq. 1), the reduce-scattered sender
gradient and the local edge gradients (App. C Eq. C1), and the all-reduced
ladder weight gradients (Sec. 5 Eq. 2) equal the single-rank results --
edge indexing exactly, values to 1e-12."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from cartesian_tensor_products_b200 import shard as S  # noqa: E402


def free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


# --------------------------------------------------------------------------
# the partition (no process group needed)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("degrees,world", [([3] * 10, 2), ([0, 9, 1, 1, 0, 4, 4, 0], 3),
                                           ([5, 5], 4), ([], 2), ([0, 0, 0], 2)])
def test_receiver_ranges_cover_and_balance(degrees, world):
    rowptr = np.concatenate([[0], np.cumsum(degrees)]).astype(np.int64)
    b = S.receiver_ranges(rowptr, world)
    N = len(degrees)
    assert len(b) == world + 1 and b[0] == 0 and b[-1] == N
    assert all(b[i] <= b[i + 1] for i in range(world))
    E = rowptr[-1]
    if E:
        per = [rowptr[b[i + 1]] - rowptr[b[i]] for i in range(world)]
        assert sum(per) == E
        assert max(per) <= E / world + max(degrees)


def test_graph_shard_local_indexing():
    from cartesian_tensor_products_b200 import workloads as W
    _, ei, _ = W.random_graph(40, 5, 6.0, 3)
    full_recv, full_send = ei
    seen = []
    for r in range(3):
        sh = S.GraphShard(ei, 40, r, 3)
        le = sh.edge_index
        assert le.dtype == np.int32
        assert np.all((le[0] >= 0) & (le[0] < sh.n_local))
        np.testing.assert_array_equal(le[0] + sh.u0, full_recv[sh.e0:sh.e1])
        np.testing.assert_array_equal(le[1], full_send[sh.e0:sh.e1])
        seen.append((sh.e0, sh.e1, sh.u0, sh.u1))
    assert seen[0][0] == 0 and seen[-1][1] == ei.shape[1]
    assert all(seen[i][1] == seen[i + 1][0] and seen[i][3] == seen[i + 1][2] for i in range(2))


# --------------------------------------------------------------------------
# world size 2 with the oracle as the per-range compute
# --------------------------------------------------------------------------

L, C, N = 2, 4, 23


def oracle_conv_fn(edge_index, edge_vec, x_all, w, n_local):
    from oracle import oracle as O
    n_all = x_all.shape[0]
    z = O.edge_conv(L, L, L, C, edge_index, edge_vec.numpy(), x_all.numpy(), w.numpy(), n_all)
    return torch.from_numpy(z[:n_local])


def oracle_vjp_fn(edge_index, edge_vec, x_all, w, g_local, n_local):
    from oracle import oracle as O
    n_all = x_all.shape[0]
    g = np.zeros((n_all, g_local.shape[1]))
    g[:n_local] = g_local.numpy()
    xb, wb, rb = O.edge_conv_vjp(L, L, L, C, edge_index, edge_vec.numpy(), x_all.numpy(),
                                 w.numpy(), g, n_all)
    return torch.from_numpy(xb), torch.from_numpy(wb), torch.from_numpy(rb)


def _inputs():
    from cartesian_tensor_products_b200 import workloads as W
    from tests.parity import ragged_graph
    degrees = [3, 0, 7, 1, 4, 4, 0, 2, 9, 3, 3, 1, 0, 5, 2, 2, 6, 1, 3, 0, 4, 2, 3]
    ei, ev = ragged_graph(N, degrees, 5.0, 31)
    d = W.conv_inputs(N, ei, L, C, 32, with_grad=True)
    lad = W.ladder_inputs(N, 2, C, 3, 33)
    return ei, ev, d, lad


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from datetime import timedelta
    from oracle import oracle as O
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    try:
        ei, ev, d, lad = _inputs()
        sh = S.GraphShard(ei, N, rank, world)
        x_local = torch.from_numpy(sh.local_nodes(d["x"]).astype(np.float64))
        ev_local = torch.from_numpy(sh.local_edges(ev))
        w_local = torch.from_numpy(sh.local_edges(d["w"]))
        z_local = S.conv_forward(sh, oracle_conv_fn, x_local, ev_local, w_local)
        g_local = torch.from_numpy(sh.local_nodes(d["g"]).astype(np.float64))
        xb_local, wb_local, rb_local = S.conv_vjp(sh, oracle_vjp_fn, x_local, ev_local, w_local,
                                                  g_local)
        # ladder: the same node ranges, node-local compute, weight gradients all-reduced
        a1 = sh.local_nodes(lad["A1"])
        gz = sh.local_nodes(lad["gz"])

        def lvjp(A1_local, gz_local):
            a, p, m = O.ladder_vjp(2, C, 3, A1_local, lad["path_w"], lad["mix_w"], gz_local)
            return torch.from_numpy(a), torch.from_numpy(p), torch.from_numpy(m)
        a1b, pwb, mwb = S.ladder_vjp(sh, lvjp, a1, gz)
        out.put((rank, sh.u0, sh.u1, sh.e0, sh.e1, sh.edge_index, z_local.numpy(),
                 xb_local.numpy(), wb_local.numpy(), rb_local.numpy(), a1b.numpy(),
                 pwb.numpy(), mwb.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_sharded_conv_vjp_and_ladder_world2():
    from oracle import oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(2)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ei, ev, d, lad = _inputs()
    z = O.edge_conv(L, L, L, C, ei, ev, d["x"], d["w"], N)
    xb, wb, rb = O.edge_conv_vjp(L, L, L, C, ei, ev, d["x"], d["w"], d["g"], N)
    a1b, pwb, mwb = O.ladder_vjp(2, C, 3, lad["A1"], lad["path_w"], lad["mix_w"], lad["gz"])
    # both ranks own receivers and edges
    assert all(r[2] > r[1] and r[4] > r[3] for r in res)
    # edge indexing: the local lists reassemble the global one exactly
    recv = np.concatenate([r[5][0] + r[1] for r in res])
    send = np.concatenate([r[5][1] for r in res])
    np.testing.assert_array_equal(np.stack([recv, send]), ei)
    tol = dict(rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(np.concatenate([r[6] for r in res]), z, **tol)
    np.testing.assert_allclose(np.concatenate([r[7] for r in res]), xb, **tol)
    np.testing.assert_allclose(np.concatenate([r[8] for r in res]), wb, **tol)
    np.testing.assert_allclose(np.concatenate([r[9] for r in res]), rb, **tol)
    np.testing.assert_allclose(np.concatenate([r[10] for r in res]), a1b, **tol)
    for r in res:        # every rank holds the summed weight gradients
        np.testing.assert_allclose(r[11], pwb, **tol)
        np.testing.assert_allclose(r[12], mwb, **tol)
