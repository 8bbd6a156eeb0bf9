"""Seeded synthetic inputs for the edge convolution and the product ladder.

This module only draws random numbers and builds graphs; it holds none of the
tensor-product arithmetic, so the CUDA path and the FP64 reference can both
read it.  Every array is float32/int32 as the library consumes it.

Workloads (shapes follow the FlashCart pages, arXiv 2610.06409):
  tiny        32 nodes in a 4 A cube, 4 random neighbours each, 8 channels,
              rank 2 (sanity case).
  microbench  1024 nodes in a 20 A cube, 128 random neighbours each,
              128 channels, rank 3 -- the Sec. 6 / App. F edge-convolution
              microbenchmark shape (1024 nodes, 128 neighbours, 128 channels).
  tiny_r4     the tiny graph with rank-4 features, directions and outputs
              plus an upstream gradient (VJP case).
  ladder      4096 nodes, 128 channels, rank 3, order 4 (Sec. 6 node-local
              benchmark shape).
  diamond     5x5x5 conventional diamond cells (a = 3.567 A, 1000 atoms),
              positions jittered, periodic 5 A neighbour list (App. F
              "Runtime and memory measurements").

Random numbers: numpy Generator(PCG64(seed)); normals are drawn as float32
directly (ziggurat) to keep the 1.5 GB weight tensors cheap to make.
"""
import numpy as np


def path_count(lin, ledge, lout):
    """Number of admissible (l1 <= lin, l2 <= ledge) -> l3 <= lout paths with
    l1 + l2 + l3 even and |l1 - l2| <= l3 <= l1 + l2 (Sec. 2)."""
    n = 0
    for l3 in range(lout + 1):
        for l1 in range(lin + 1):
            for l2 in range(ledge + 1):
                if abs(l1 - l2) <= l3 <= l1 + l2 and (l1 + l2 + l3) % 2 == 0:
                    n += 1
    return n


def paths_per_rank(lin, ledge, lout):
    out = [0] * (lout + 1)
    for l3 in range(lout + 1):
        for l1 in range(lin + 1):
            for l2 in range(ledge + 1):
                if abs(l1 - l2) <= l3 <= l1 + l2 and (l1 + l2 + l3) % 2 == 0:
                    out[l3] += 1
    return out


def rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def normal(g, shape, scale=1.0):
    a = g.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        a *= np.float32(scale)
    return a


def random_graph(n_nodes, k, box, seed):
    """n_nodes positions uniform in [0, box)^3 and, for every receiver u, k
    distinct random senders v != u.  Edges are receiver-major with senders
    ascending inside each receiver.  edge_vec = pos[v] - pos[u] (Sec. 2: the
    edge vector points from the receiver to its neighbour)."""
    g = rng(seed)
    pos = g.uniform(0.0, box, size=(n_nodes, 3))
    recv = np.repeat(np.arange(n_nodes, dtype=np.int64), k)
    send = np.empty(n_nodes * k, dtype=np.int64)
    for u in range(n_nodes):
        s = g.choice(n_nodes - 1, size=k, replace=False)
        s = np.where(s >= u, s + 1, s)
        send[u * k:(u + 1) * k] = np.sort(s)
    edge_index = np.stack([recv, send]).astype(np.int32)
    edge_vec = (pos[send] - pos[recv]).astype(np.float32)
    return pos.astype(np.float32), edge_index, edge_vec


def conv_inputs(n_nodes, edge_index, lmax, channels, seed, with_grad=False,
                sum_paths=False):
    """Node features (N(0,1) per independent component), per-edge/path/channel
    weights N(0,1)/sqrt(#paths) and, optionally, an N(0,1) upstream gradient
    shaped like the output."""
    g = rng(seed)
    E = edge_index.shape[1]
    P = path_count(lmax, lmax, lmax)
    x = normal(g, (n_nodes, (lmax + 1) ** 2 * channels))
    w = normal(g, (E, P, channels), 1.0 / np.sqrt(P))
    out = {"x": x, "w": w}
    if with_grad:
        if sum_paths:
            zr = (lmax + 1) ** 2
        else:
            zr = sum((2 * l + 1) * p
                     for l, p in enumerate(paths_per_rank(lmax, lmax, lmax)))
        out["g"] = normal(g, (n_nodes, zr * channels))
    return out


def cotangents(n_nodes, n_edges, lmax, channels, seed, edge_vec=None):
    """Cotangents of the VJP outputs for the VJP-of-VJP (App. C Eq. C2):
    vx like x_bar (N(0,1)), vw like w_bar (N(0,1)/sqrt(#paths)) and vr like
    r_bar (N(0,1) per edge, scaled by |r| when edge vectors are given, so a
    unit relative step along vr is a unit relative step of the edge)."""
    g = rng(seed)
    P = path_count(lmax, lmax, lmax)
    vx = normal(g, (n_nodes, (lmax + 1) ** 2 * channels))
    vw = normal(g, (n_edges, P, channels), 1.0 / np.sqrt(P))
    vr = normal(g, (n_edges, 3))
    if edge_vec is not None:
        vr = (vr * np.linalg.norm(np.asarray(edge_vec, np.float64), axis=1)[:, None]).astype(np.float32)
    return {"vx": vx, "vw": vw, "vr": vr}


def tiny(seed=1):
    pos, ei, ev = random_graph(32, 4, 4.0, seed)
    d = conv_inputs(32, ei, 2, 8, seed + 100)
    return dict(name="tiny", n_nodes=32, lmax=2, channels=8, pos=pos,
                edge_index=ei, edge_vec=ev, **d)


def microbench(seed=2, lmax=3, weight_seed=None):
    pos, ei, ev = random_graph(1024, 128, 20.0, seed)
    d = conv_inputs(1024, ei, lmax, 128,
                    (seed + 100) if weight_seed is None else weight_seed,
                    with_grad=(lmax == 4))
    return dict(name="microbench" if lmax == 3 else "microbench_r%d" % lmax,
                n_nodes=1024, lmax=lmax, channels=128, pos=pos,
                edge_index=ei, edge_vec=ev, **d)


def sharded_microbench(rank, world, n_per_rank=1024, k=128, channels=128, lmax=3, seed=2):
    """One graph of world x n_per_rank nodes spread over `world` ranks by
    receiver range (weak scaling: every rank owns n_per_rank receivers with
    k random distinct senders among ALL nodes, the microbenchmark's per-rank
    shape).  Positions are uniform in a cube that keeps the microbenchmark's
    density; receiver block b draws its senders from seed + 1000 b, so every
    rank builds the same global edge list.  Returns the global edge_index
    and bounds, and this rank's own node features, edge vectors and weights
    (rank-seeded)."""
    n = world * n_per_rank
    box = 20.0 * world ** (1.0 / 3.0)
    pos = rng(seed).uniform(0.0, box, size=(n, 3))
    recv = np.repeat(np.arange(n, dtype=np.int64), k)
    send = np.empty(n * k, dtype=np.int64)
    for b in range(world):
        g = rng(seed + 1000 * b)
        for u in range(b * n_per_rank, (b + 1) * n_per_rank):
            s = g.choice(n - 1, size=k, replace=False)
            s = np.where(s >= u, s + 1, s)
            send[u * k:(u + 1) * k] = np.sort(s)
    edge_index = np.stack([recv, send]).astype(np.int32)
    e0, e1 = rank * n_per_rank * k, (rank + 1) * n_per_rank * k
    ev = (pos[send[e0:e1]] - pos[recv[e0:e1]]).astype(np.float32)
    g = rng(seed + 100 + 7919 * rank)
    P = path_count(lmax, lmax, lmax)
    x = normal(g, (n_per_rank, (lmax + 1) ** 2 * channels))
    w = normal(g, (e1 - e0, P, channels), 1.0 / np.sqrt(P))
    return dict(name="microbench_sharded", n_nodes=n, lmax=lmax, channels=channels,
                edge_index=edge_index, bounds=[b * n_per_rank for b in range(world + 1)],
                x_local=x, w_local=w, edge_vec_local=ev)


def microbench_grad(seed=2, lmax=3, weight_seed=None):
    """The microbenchmark graph with an upstream gradient (VJP rows)."""
    pos, ei, ev = random_graph(1024, 128, 20.0, seed)
    d = conv_inputs(1024, ei, lmax, 128,
                    (seed + 100) if weight_seed is None else weight_seed,
                    with_grad=True)
    return dict(name="microbench_vjp_r%d" % lmax, n_nodes=1024, lmax=lmax,
                channels=128, pos=pos, edge_index=ei, edge_vec=ev, **d)


def tiny_r4(seed=1, feature_seed=3):
    pos, ei, ev = random_graph(32, 4, 4.0, seed)
    d = conv_inputs(32, ei, 4, 8, feature_seed, with_grad=True)
    return dict(name="tiny_r4", n_nodes=32, lmax=4, channels=8, pos=pos,
                edge_index=ei, edge_vec=ev, **d)


def ladder_inputs(n_nodes, lmax, channels, order, seed):
    """A_1 ~ N(0,1); path weights W_v ~ N(0,1)/sqrt(P_l3) for the output rank
    of each path; per-rank mixing matrices ~ N(0, 1/channels); gz ~ N(0,1)."""
    g = rng(seed)
    ppr = paths_per_rank(lmax, lmax, lmax)
    l3_of_path = []
    for l3 in range(lmax + 1):
        l3_of_path += [l3] * ppr[l3]
    scale = np.array([1.0 / np.sqrt(ppr[l3]) for l3 in l3_of_path],
                     dtype=np.float32)
    S = order - 1
    A1 = normal(g, (n_nodes, (lmax + 1) ** 2 * channels))
    path_w = normal(g, (S, len(l3_of_path), channels)) * scale[None, :, None]
    mix_w = normal(g, (S, lmax + 1, channels, channels),
                   1.0 / np.sqrt(channels))
    gz = normal(g, (n_nodes, (lmax + 1) ** 2 * channels))
    return dict(A1=A1, path_w=np.ascontiguousarray(path_w), mix_w=mix_w, gz=gz)


def full_ladder_inputs(n_nodes, lmax, channels, order, seed):
    """Full ladder (Sec. 5 Eq. 2): A ~ N(0,1); W1 ~ N(0, 1/C) per rank;
    for each later step and rank l a [C][P_l C] map ~ N(0, 1/(P_l C)),
    stored rank after rank; gz ~ N(0,1)."""
    g = rng(seed)
    ppr = paths_per_rank(lmax, lmax, lmax)
    P = sum(ppr)
    C = channels
    A = normal(g, (n_nodes, (lmax + 1) ** 2 * C))
    W1 = normal(g, (lmax + 1, C, C), 1.0 / np.sqrt(C))
    blocks = []
    for q in range(order - 1):
        blocks.append(np.concatenate([normal(g, (C, p * C), 1.0 / np.sqrt(p * C)).ravel()
                                      for p in ppr]))
    Wq = np.stack(blocks) if blocks else np.zeros((0, C * P * C), np.float32)
    gz = normal(g, (n_nodes, (lmax + 1) ** 2 * C))
    return dict(A=A, W1=W1, Wq=np.ascontiguousarray(Wq, dtype=np.float32), gz=gz)


def ladder(seed=4, n_nodes=4096, channels=128, lmax=3, order=4):
    d = ladder_inputs(n_nodes, lmax, channels, order, seed)
    return dict(name="ladder", n_nodes=n_nodes, lmax=lmax, channels=channels,
                order=order, **d)


DIAMOND_BASIS = np.array([
    [0.0, 0.0, 0.0], [0.0, 0.5, 0.5], [0.5, 0.0, 0.5], [0.5, 0.5, 0.0],
    [0.25, 0.25, 0.25], [0.25, 0.75, 0.75], [0.75, 0.25, 0.75],
    [0.75, 0.75, 0.25]])


def diamond_positions(cells=5, a=3.567, jitter=0.05, seed=5):
    g = rng(seed)
    grid = np.stack(np.meshgrid(np.arange(cells), np.arange(cells),
                                np.arange(cells), indexing="ij"), -1)
    grid = grid.reshape(-1, 1, 3)
    pos = (grid + DIAMOND_BASIS[None]) .reshape(-1, 3) * a
    pos = pos + g.normal(0.0, jitter, size=pos.shape)
    box = cells * a
    return pos, box


def periodic_neighbours(pos, box, cutoff):
    """All ordered pairs (u, v), v != u, whose minimum-image distance is below
    the cutoff (exact when the box exceeds twice the cutoff).  Receiver-major,
    senders ascending; edge_vec = minimum image of pos[v] - pos[u]."""
    assert box > 2 * cutoff
    n = pos.shape[0]
    recv, send, vecs = [], [], []
    for u in range(n):
        d = pos - pos[u]
        d -= box * np.round(d / box)
        r2 = np.einsum("ij,ij->i", d, d)
        nb = np.nonzero((r2 < cutoff * cutoff) & (np.arange(n) != u))[0]
        recv.append(np.full(nb.shape, u))
        send.append(nb)
        vecs.append(d[nb])
    ei = np.stack([np.concatenate(recv), np.concatenate(send)]).astype(np.int32)
    ev = np.concatenate(vecs).astype(np.float32)
    return ei, ev


def diamond(seed=5, channels=128, lmax=3, order=5, cutoff=5.0, cells=5):
    """Full interaction block workload: diamond cell, periodic neighbour list,
    node features, per-(edge, path, channel) weights omega ~ N(0,1)/sqrt(P)
    (multiplied in the block by the cosine envelope and 1/sqrt(mean
    neighbours)), ladder weights.  shift = edge_vec - (pos[v] - pos[u])."""
    pos, box = diamond_positions(cells=cells, seed=seed)
    ei, ev = periodic_neighbours(pos, box, cutoff)
    n = pos.shape[0]
    g = rng(seed + 100)
    P = path_count(lmax, lmax, lmax)
    E = ei.shape[1]
    x = normal(g, (n, (lmax + 1) ** 2 * channels))
    omega = normal(g, (E, P, channels), 1.0 / np.sqrt(P))
    lad = ladder_inputs(n, lmax, channels, order, seed + 200)
    shift = (ev.astype(np.float64) - (pos[ei[1]] - pos[ei[0]]))
    shift = box * np.round(shift / box)
    return dict(name="diamond", n_nodes=n, lmax=lmax, channels=channels,
                order=order, cutoff=cutoff, box=box, pos=pos.astype(np.float32),
                pos64=pos, edge_index=ei, edge_vec=ev, shift=shift, x=x, omega=omega,
                path_w=lad["path_w"], mix_w=lad["mix_w"],
                edge_scale=float(1.0 / np.sqrt(ei.shape[1] / n)))
