"""ctypes front end of the FP64 oracle (fc_oracle.c).

TEST INFRASTRUCTURE ONLY.  Inputs are promoted to float64 and made
contiguous here; every computation happens in the C source, which follows
the FlashCart pages (arXiv 2610.06409) as cited there.
"""
import ctypes as ct
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ct.CDLL(path)
        d = ct.POINTER(ct.c_double)
        i32 = ct.POINTER(ct.c_int32)
        ip = ct.POINTER(ct.c_int)
        u8 = ct.POINTER(ct.c_ubyte)
        sig = {
            "orc_permavg": (None, [ct.c_int, d, d]),
            "orc_detrace": (None, [ct.c_int, d, d]),
            "orc_stf_dense": (None, [ct.c_int, d, d]),
            "orc_stf_extract": (None, [ct.c_int, d, d]),
            "orc_comp_pxyz": (None, [ct.c_int, ct.c_int, ip, ip, ip]),
            "orc_direction_dense": (None, [ct.c_int, d, d]),
            "orc_direction": (None, [ct.c_int, d, d]),
            "orc_direction_jac": (None, [ct.c_int, d, d]),
            "orc_admissible": (ct.c_int, [ct.c_int] * 3),
            "orc_path_norm": (ct.c_double, [ct.c_int] * 3),
            "orc_product_dense": (ct.c_int, [ct.c_int] * 3 + [d, d, d, ct.c_int]),
            "orc_product": (ct.c_int, [ct.c_int] * 3 + [d, d, d]),
            "orc_path_coeffs": (None, [ct.c_int] * 3 + [d]),
            "orc_paths": (ct.c_int, [ct.c_int] * 3 + [ip, ip, ip]),
            "orc_edge_conv": (ct.c_int, [ct.c_int] * 7 + [i32, i32, d, d, d, u8, d]),
            "orc_edge_conv_vjp": (ct.c_int, [ct.c_int] * 7 + [i32, i32, d, d, d, d, u8, d, d, d]),
            "orc_edge_conv_odd": (ct.c_int, [ct.c_int] * 7 + [i32, i32, d, d, d, u8, d]),
            "orc_edge_conv_odd_vjp": (ct.c_int, [ct.c_int] * 7 + [i32, i32, d, d, d, d, u8, d, d,
                                                                  d]),
            "orc_odd_admissible": (ct.c_int, [ct.c_int] * 3),
            "orc_product_odd_dense": (ct.c_int, [ct.c_int] * 3 + [d, d, d]),
            "orc_product_odd": (ct.c_int, [ct.c_int] * 3 + [d, d, d]),
            "orc_path_coeffs_odd": (None, [ct.c_int] * 3 + [d]),
            "orc_paths_odd": (ct.c_int, [ct.c_int] * 3 + [ip, ip, ip]),
            "orc_edge_conv_vjp2": (ct.c_int, [ct.c_int] * 7 + [i32, i32, d, d, d, d, d, d, d, u8,
                                                               d, d, d, d]),
            "orc_direction_hvp": (None, [ct.c_int, d, d, d, d]),
            "orc_full_ladder": (ct.c_int, [ct.c_int] * 4 + [d, d, d, u8, d, d]),
            "orc_full_ladder_vjp": (ct.c_int, [ct.c_int] * 4 + [d, d, d, d, u8, d, d, d]),
            "orc_ladder": (ct.c_int, [ct.c_int] * 4 + [d, d, d, u8, d, d]),
            "orc_ladder_vjp": (ct.c_int, [ct.c_int] * 4 + [d, d, d, d, u8, d, d, d]),
            "orc_max_rank": (ct.c_int, []),
            "orc_num_threads": (ct.c_int, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _d(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _pd(a):
    if a is None:
        return None
    return a.ctypes.data_as(ct.POINTER(ct.c_double))


def _pi32(a):
    return a.ctypes.data_as(ct.POINTER(ct.c_int32))


def _pu8(a):
    if a is None:
        return None
    return a.ctypes.data_as(ct.POINTER(ct.c_ubyte))


def _mask(m, n):
    if m is None:
        return None
    m = np.ascontiguousarray(np.asarray(m, dtype=np.uint8))
    assert m.shape == (n,)
    return m


# --------------------------------------------------------------------------
# tensors
# --------------------------------------------------------------------------

def permavg(l, t):
    t = _d(t).reshape(-1)
    out = np.empty(3 ** l)
    lib().orc_permavg(l, _pd(t), _pd(out))
    return out.reshape((3,) * l)


def detrace(l, t):
    t = _d(t).reshape(-1)
    out = np.empty(3 ** l)
    lib().orc_detrace(l, _pd(t), _pd(out))
    return out.reshape((3,) * l)


def stf_dense(l, comps):
    c = _d(comps)
    assert c.shape == (2 * l + 1,)
    out = np.empty(3 ** l)
    lib().orc_stf_dense(l, _pd(c), _pd(out))
    return out.reshape((3,) * l)


def stf_extract(l, dense):
    t = _d(dense).reshape(-1)
    out = np.empty(2 * l + 1)
    lib().orc_stf_extract(l, _pd(t), _pd(out))
    return out


def comp_pxyz(l, c):
    a, b, z = ct.c_int(), ct.c_int(), ct.c_int()
    lib().orc_comp_pxyz(l, c, ct.byref(a), ct.byref(b), ct.byref(z))
    return a.value, b.value, z.value


def direction_dense(l, r):
    r = _d(r)
    out = np.empty(3 ** l)
    lib().orc_direction_dense(l, _pd(r), _pd(out))
    return out.reshape((3,) * l)


def direction(l, r):
    r = _d(r)
    out = np.empty(2 * l + 1)
    lib().orc_direction(l, _pd(r), _pd(out))
    return out


def direction_jac(l, r):
    r = _d(r)
    out = np.empty((2 * l + 1) * 3)
    lib().orc_direction_jac(l, _pd(r), _pd(out))
    return out.reshape(2 * l + 1, 3)


def direction_hvp(l, r, ybar, v):
    """(d^2 <ybar, T_l(r/|r|)> / dr dr) v, exact (App. C, derivatives of the
    direction tensors used in force training)."""
    out = np.empty(3)
    lib().orc_direction_hvp(l, _pd(_d(r)), _pd(_d(ybar)), _pd(_d(v)), _pd(out))
    return out


def admissible(l1, l2, l3):
    return bool(lib().orc_admissible(l1, l2, l3))


def path_norm(l1, l2, l3):
    return lib().orc_path_norm(l1, l2, l3)


def product_dense(l1, l2, l3, x, y, route=0):
    x, y = _d(x), _d(y)
    out = np.empty(3 ** l3)
    rc = lib().orc_product_dense(l1, l2, l3, _pd(x), _pd(y), _pd(out), route)
    if rc:
        raise ValueError("path (%d,%d)->%d not admissible" % (l1, l2, l3))
    return out.reshape((3,) * l3)


def product(l1, l2, l3, x, y):
    x, y = _d(x), _d(y)
    out = np.empty(2 * l3 + 1)
    rc = lib().orc_product(l1, l2, l3, _pd(x), _pd(y), _pd(out))
    if rc:
        raise ValueError("path (%d,%d)->%d not admissible" % (l1, l2, l3))
    return out


def path_coeffs(l1, l2, l3):
    out = np.empty((2 * l3 + 1) * (2 * l1 + 1) * (2 * l2 + 1))
    lib().orc_path_coeffs(l1, l2, l3, _pd(out))
    return out.reshape(2 * l3 + 1, 2 * l1 + 1, 2 * l2 + 1)


def paths(lin, ledge, lout, odd=False):
    """Admissible paths ordered by l3, then l1, then l2; odd=True lists the
    odd-J (Levi-Civita) paths instead."""
    f = lib().orc_paths_odd if odd else lib().orc_paths
    n = f(lin, ledge, lout, None, None, None)
    a = (ct.c_int * max(n, 1))()
    b = (ct.c_int * max(n, 1))()
    c = (ct.c_int * max(n, 1))()
    f(lin, ledge, lout, a, b, c)
    return [(a[i], b[i], c[i]) for i in range(n)]


# --------------------------------------------------------------------------
# odd-J products (App. B after Eq. B1; Sec. 7): one Levi-Civita contraction
# --------------------------------------------------------------------------

def odd_admissible(l1, l2, l3):
    return bool(lib().orc_odd_admissible(l1, l2, l3))


def product_odd_dense(l1, l2, l3, x, y):
    x, y = _d(x), _d(y)
    out = np.empty(3 ** l3)
    if lib().orc_product_odd_dense(l1, l2, l3, _pd(x), _pd(y), _pd(out)):
        raise ValueError("path (%d,%d)->%d is not an odd-J path" % (l1, l2, l3))
    return out.reshape((3,) * l3)


def product_odd(l1, l2, l3, x, y):
    x, y = _d(x), _d(y)
    out = np.empty(2 * l3 + 1)
    if lib().orc_product_odd(l1, l2, l3, _pd(x), _pd(y), _pd(out)):
        raise ValueError("path (%d,%d)->%d is not an odd-J path" % (l1, l2, l3))
    return out


def path_coeffs_odd(l1, l2, l3):
    out = np.empty((2 * l3 + 1) * (2 * l1 + 1) * (2 * l2 + 1))
    lib().orc_path_coeffs_odd(l1, l2, l3, _pd(out))
    return out.reshape(2 * l3 + 1, 2 * l1 + 1, 2 * l2 + 1)


def num_threads():
    return lib().orc_num_threads()


# --------------------------------------------------------------------------
# edge convolution (Sec. 4 Eq. 1) and its VJP (App. C Eq. C1)
# --------------------------------------------------------------------------

def zrow(lin, ledge, lout, sum_paths=False, odd=False):
    """Output row length / C for the edge convolution."""
    ps = paths(lin, ledge, lout, odd)
    if sum_paths:
        return (lout + 1) ** 2
    return sum(2 * l3 + 1 for (_, _, l3) in ps)


def edge_conv(lin, ledge, lout, C, edge_index, edge_vec, x, w, n_nodes,
              sum_paths=False, recv_mask=None, odd=False):
    """z = Eq. (1).  With recv_mask, only the listed receivers' rows are
    computed (their edges are selected here; other rows stay zero).
    odd=True: over the odd-J paths (pseudo-tensor outputs)."""
    ei = np.asarray(edge_index)
    P = len(paths(lin, ledge, lout, odd))
    if recv_mask is not None:
        m = _mask(recv_mask, n_nodes)
        sel = np.nonzero(m[ei[0]])[0]
        ei, edge_vec, w = ei[:, sel], np.asarray(edge_vec)[sel], np.asarray(w)[sel]
    ei = np.ascontiguousarray(ei, dtype=np.int32)
    E = ei.shape[1]
    recv = np.ascontiguousarray(ei[0])
    send = np.ascontiguousarray(ei[1])
    vec = _d(edge_vec).reshape(E, 3)
    x = _d(x)
    w = _d(w).reshape(E, P, C)
    assert x.shape == (n_nodes, (lin + 1) ** 2 * C)
    zr = zrow(lin, ledge, lout, sum_paths, odd)
    z = np.empty((n_nodes, zr * C))
    f = lib().orc_edge_conv_odd if odd else lib().orc_edge_conv
    rc = f(lin, ledge, lout, C, int(sum_paths), n_nodes, E,
                             _pi32(recv), _pi32(send), _pd(vec), _pd(x), _pd(w),
                             None, _pd(z))
    assert rc == 0
    return z


def edge_conv_vjp(lin, ledge, lout, C, edge_index, edge_vec, x, w, g, n_nodes,
                  sum_paths=False, edge_mask=None, want=("x", "w", "r"), odd=False):
    """Eq. (C1) summed over edges.  With edge_mask, only the listed edges
    contribute (they are selected here); w_bar / r_bar rows of the other
    edges are zero.  odd=True: the VJP of the odd-J convolution."""
    ei_full = np.asarray(edge_index)
    E_full = ei_full.shape[1]
    P = len(paths(lin, ledge, lout, odd))
    sel = None
    ei, ev, ww = ei_full, np.asarray(edge_vec), np.asarray(w)
    if edge_mask is not None:
        sel = np.nonzero(_mask(edge_mask, E_full))[0]
        ei, ev, ww = ei[:, sel], ev[sel], ww[sel]
    ei = np.ascontiguousarray(ei, dtype=np.int32)
    E = ei.shape[1]
    recv = np.ascontiguousarray(ei[0])
    send = np.ascontiguousarray(ei[1])
    vec = _d(ev).reshape(E, 3)
    x, ww, g = _d(x), _d(ww).reshape(E, P, C), _d(g)
    xb = np.empty(((n_nodes, (lin + 1) ** 2 * C))) if "x" in want else None
    wb = np.empty((E, P, C)) if "w" in want else None
    rb = np.empty((E, 3)) if "r" in want else None
    f = lib().orc_edge_conv_odd_vjp if odd else lib().orc_edge_conv_vjp
    rc = f(lin, ledge, lout, C, int(sum_paths), n_nodes, E,
                                 _pi32(recv), _pi32(send), _pd(vec), _pd(x),
                                 _pd(ww), _pd(g), None, _pd(xb), _pd(wb), _pd(rb))
    assert rc == 0
    if sel is not None:
        if wb is not None:
            full = np.zeros((E_full, P, C)); full[sel] = wb; wb = full
        if rb is not None:
            full = np.zeros((E_full, 3)); full[sel] = rb; rb = full
    return xb, wb, rb


def edge_conv_vjp_vjp(lin, ledge, lout, C, edge_index, edge_vec, x, w, g, vx, vw, vr,
                      n_nodes, sum_paths=False, edge_mask=None, want=("g", "x", "w", "r")):
    """VJP-of-VJP (App. C Eq. C2, Algorithm 3): gradients of
    <vx, x_bar> + <vw, w_bar> + <vr, r_bar> with respect to (g, x, w, edge
    vectors), where (x_bar, w_bar, r_bar) = edge_conv_vjp(...).  vx, vw, vr
    may be None (zero cotangent).  With edge_mask only the listed edges
    contribute; w_hat / r_hat rows of the other edges are zero."""
    ei_full = np.asarray(edge_index)
    E_full = ei_full.shape[1]
    P = len(paths(lin, ledge, lout))
    sel = None
    ei, ev, ww = ei_full, np.asarray(edge_vec), np.asarray(w)
    vww = None if vw is None else np.asarray(vw)
    vrr = None if vr is None else np.asarray(vr)
    if edge_mask is not None:
        sel = np.nonzero(_mask(edge_mask, E_full))[0]
        ei, ev, ww = ei[:, sel], ev[sel], ww[sel]
        vww = None if vww is None else vww[sel]
        vrr = None if vrr is None else vrr[sel]
    ei = np.ascontiguousarray(ei, dtype=np.int32)
    E = ei.shape[1]
    recv = np.ascontiguousarray(ei[0])
    send = np.ascontiguousarray(ei[1])
    vec = _d(ev).reshape(E, 3)
    x, ww, g = _d(x), _d(ww).reshape(E, P, C), _d(g)
    vx = None if vx is None else _d(vx)
    vww = None if vww is None else _d(vww).reshape(E, P, C)
    vrr = None if vrr is None else _d(vrr).reshape(E, 3)
    zrow = g.shape[1] // C
    gh = np.empty((n_nodes, zrow * C)) if "g" in want else None
    xh = np.empty((n_nodes, (lin + 1) ** 2 * C)) if "x" in want else None
    wh = np.empty((E, P, C)) if "w" in want else None
    rh = np.empty((E, 3)) if "r" in want else None
    rc = lib().orc_edge_conv_vjp2(lin, ledge, lout, C, int(sum_paths), n_nodes, E,
                                  _pi32(recv), _pi32(send), _pd(vec), _pd(x), _pd(ww),
                                  _pd(g), _pd(vx), _pd(vww), _pd(vrr), None,
                                  _pd(gh), _pd(xh), _pd(wh), _pd(rh))
    assert rc == 0
    if sel is not None:
        if wh is not None:
            full = np.zeros((E_full, P, C)); full[sel] = wh; wh = full
        if rh is not None:
            full = np.zeros((E_full, 3)); full[sel] = rh; rh = full
    return gh, xh, wh, rh


# --------------------------------------------------------------------------
# node-local ladder (Sec. 5 Eq. 2, path-reduced products + per-rank mixing)
# --------------------------------------------------------------------------

def ladder(L, C, order, A1, path_w, mix_w, node_mask=None):
    A1 = _d(A1)
    N = A1.shape[0]
    P = len(paths(L, L, L))
    path_w = _d(path_w).reshape(max(order - 1, 0), P, C)
    mix_w = _d(mix_w).reshape(max(order - 1, 0), L + 1, C, C)
    states = np.empty((max(order - 1, 0), N, (L + 1) ** 2 * C))
    z = np.empty((N, (L + 1) ** 2 * C))
    m = _mask(node_mask, N)
    rc = lib().orc_ladder(L, C, order, N, _pd(A1), _pd(path_w), _pd(mix_w),
                          _pu8(m), _pd(states), _pd(z))
    assert rc == 0
    return states, z


def ladder_vjp(L, C, order, A1, path_w, mix_w, gz, node_mask=None):
    A1 = _d(A1)
    N = A1.shape[0]
    P = len(paths(L, L, L))
    path_w = _d(path_w).reshape(max(order - 1, 0), P, C)
    mix_w = _d(mix_w).reshape(max(order - 1, 0), L + 1, C, C)
    gz = _d(gz)
    A1b = np.empty_like(A1)
    pwb = np.zeros_like(path_w)
    mxb = np.zeros_like(mix_w)
    m = _mask(node_mask, N)
    rc = lib().orc_ladder_vjp(L, C, order, N, _pd(A1), _pd(path_w), _pd(mix_w),
                              _pd(gz), _pu8(m), _pd(A1b), _pd(pwb), _pd(mxb))
    assert rc == 0
    return A1b, pwb, mxb


# --------------------------------------------------------------------------
# one interaction block: envelope-weighted convolution, ladder, E, forces
# --------------------------------------------------------------------------

def envelope(edge_vec, r_cut, scale):
    """s(r) = scale (cos(pi r / r_cut) + 1) / 2 for r < r_cut (else 0), and
    ds/dr: a smooth radial envelope vanishing at the cutoff (App. B)."""
    r = np.linalg.norm(np.asarray(edge_vec, dtype=np.float64), axis=1)
    inside = r < r_cut
    s = np.where(inside, 0.5 * scale * (np.cos(np.pi * r / r_cut) + 1.0), 0.0)
    sp = np.where(inside, -0.5 * scale * np.pi / r_cut * np.sin(np.pi * r / r_cut), 0.0)
    return s, sp, r


def block_energy_forces(L, C, order, edge_index, edge_vec, x, omega, path_w, mix_w,
                        n_nodes, r_cut, edge_scale, recv_mask=None):
    """E = sum over nodes and channels of the rank-0 ladder output, with the
    ladder fed by the convolution of paths summed per output rank and edge
    weights omega * s(|r|); F = -dE/dpos by the chain rule
    dE/dr_e = r_bar_T(e) + s'(|r_e|) r_hat_e sum_{p,k} omega w_bar_eff.
    With recv_mask only those receivers' energies and the gradients of their
    incoming edges are formed.  Returns (E per node, dE/dr per edge, F)."""
    ei = np.asarray(edge_index)
    ev = np.asarray(edge_vec, dtype=np.float64)
    om = np.asarray(omega, dtype=np.float64)
    s, sp, r = envelope(ev, r_cut, edge_scale)
    w_eff = om * s[:, None, None]
    A1 = edge_conv(L, L, L, C, ei, ev, x, w_eff, n_nodes, sum_paths=True,
                   recv_mask=recv_mask)
    _, z = ladder(L, C, order, A1, path_w, mix_w, node_mask=recv_mask)
    e_node = z[:, :C].sum(1)
    gz = np.zeros_like(z)
    gz[:, :C] = 1.0
    if recv_mask is not None:
        gz *= np.asarray(recv_mask, dtype=np.float64)[:, None]
    A1b, _, _ = ladder_vjp(L, C, order, A1, path_w, mix_w, gz, node_mask=recv_mask)
    emask = None if recv_mask is None else np.asarray(recv_mask)[ei[0]].astype(np.uint8)
    _, wb, rb = edge_conv_vjp(L, L, L, C, ei, ev, x, w_eff, A1b, n_nodes, sum_paths=True,
                              edge_mask=emask)
    rhat = ev / r[:, None]
    dEdr = rb + ((wb * om).sum((1, 2)) * sp)[:, None] * rhat
    F = np.zeros((n_nodes, 3))
    np.add.at(F, ei[1], -dEdr)
    np.add.at(F, ei[0], dEdr)
    return e_node, dEdr, F


def full_ladder(L, C, order, A, W1, Wq, node_mask=None):
    """Full correlation ladder (Sec. 5 Eq. 2): per-path products, each step's
    paths and channels mixed per output rank by Wq; returns (states
    [order][N][(L+1)^2 C] = phi_1..phi_order, z = their sum).  W1:
    [L+1][C][C]; Wq: [order-1][C*P*C], rank blocks [C][P_l C] in rank order."""
    A = _d(A)
    N = A.shape[0]
    P = len(paths(L, L, L))
    W1 = _d(W1).reshape(L + 1, C, C)
    Wq = _d(Wq).reshape(order - 1, C * P * C) if order > 1 else np.zeros((1, C * P * C))
    states = np.empty((order, N, (L + 1) ** 2 * C))
    z = np.empty((N, (L + 1) ** 2 * C))
    m = None if node_mask is None else _mask(node_mask, N)
    rc = lib().orc_full_ladder(L, C, order, N, _pd(A), _pd(W1), _pd(np.ascontiguousarray(Wq)),
                               None if m is None else m.ctypes.data_as(ct.POINTER(ct.c_uint8)),
                               _pd(states), _pd(z))
    assert rc == 0
    return states, z


def full_ladder_vjp(L, C, order, A, W1, Wq, gz, node_mask=None):
    """Gradients (A_bar, W1_bar, Wq_bar) of <gz, z> for the full ladder, by
    reverse accumulation through its steps (Sec. 5 Eq. 2; App. C Eq. C1 for
    each bilinear product).  Weight gradients sum over the selected nodes."""
    A = _d(A)
    N = A.shape[0]
    P = len(paths(L, L, L))
    W1 = _d(W1).reshape(L + 1, C, C)
    Wq = _d(Wq).reshape(order - 1, C * P * C) if order > 1 else np.zeros((1, C * P * C))
    gz = _d(gz)
    Ab = np.empty_like(A)
    W1b = np.zeros_like(W1)
    Wqb = np.zeros_like(Wq)
    m = None if node_mask is None else _mask(node_mask, N)
    rc = lib().orc_full_ladder_vjp(L, C, order, N, _pd(A), _pd(W1), _pd(np.ascontiguousarray(Wq)),
                                   _pd(gz), _pu8(m), _pd(Ab), _pd(W1b), _pd(Wqb))
    assert rc == 0
    return Ab, W1b, (Wqb if order > 1 else Wqb[:0])
