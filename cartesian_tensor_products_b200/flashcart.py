"""Thin ctypes binding of libflashcart (C ABI in include/flashcart.h).

Argument marshalling only: tensors are checked for device, dtype and shape,
their device pointers and the current CUDA stream are handed to the C entry
points, and a non-zero status becomes a FlashCartError.  Every step of the
computation runs in the library's CUDA kernels; there is no fallback.  If the
library has not been built this module raises on import.

Conventions (layouts, path order, component order) are those of the header.
"""
import ctypes as ct
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libflashcart.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libflashcart.so is not built (expected at %s); run "
        "`python -m cartesian_tensor_products_b200.build`" % LIB_PATH)

_lib = ct.CDLL(LIB_PATH)

FC_OK = 0


class FlashCartError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s: %s (status %d)" % (
            where, _lib.fc_status_string(status).decode(), status))


class ConvDesc(ct.Structure):
    _fields_ = [("lmax_in", ct.c_int), ("lmax_edge", ct.c_int),
                ("lmax_out", ct.c_int), ("channels", ct.c_int),
                ("sum_paths", ct.c_int), ("envelope", ct.c_int),
                ("r_cut", ct.c_float), ("edge_scale", ct.c_float)]


class LadderDesc(ct.Structure):
    _fields_ = [("lmax", ct.c_int), ("channels", ct.c_int), ("order", ct.c_int)]


_vp = ct.c_void_p
_SIGS = {
    "fc_status_string": (ct.c_char_p, [ct.c_int]),
    "fc_version": (ct.c_int, []),
    "fc_conv_num_paths": (ct.c_int, [ct.POINTER(ConvDesc)]),
    "fc_conv_out_row": (ct.c_int, [ct.POINTER(ConvDesc)]),
    "fc_conv_path": (ct.c_int, [ct.POINTER(ConvDesc), ct.c_int, ct.POINTER(ct.c_int),
                                ct.POINTER(ct.c_int), ct.POINTER(ct.c_int)]),
    "fc_build_rowptr": (ct.c_int, [ct.c_int, ct.c_int, _vp, _vp, _vp, _vp, _vp]),
    "fc_build_rowptr_rect": (ct.c_int, [ct.c_int, ct.c_int, ct.c_int, _vp, _vp, _vp, _vp, _vp]),
    "fc_edge_conv": (ct.c_int, [ct.POINTER(ConvDesc), ct.c_int, ct.c_int,
                                _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fc_edge_conv_rect": (ct.c_int, [ct.POINTER(ConvDesc), ct.c_int, ct.c_int, ct.c_int,
                                     _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fc_edge_conv_vjp": (ct.c_int, [ct.POINTER(ConvDesc), ct.c_int, ct.c_int,
                                    _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fc_edge_conv_vjp_rect": (ct.c_int, [ct.POINTER(ConvDesc), ct.c_int, ct.c_int, ct.c_int,
                                         _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fc_conv_odd_num_paths": (ct.c_int, [ct.POINTER(ConvDesc)]),
    "fc_conv_odd_out_row": (ct.c_int, [ct.POINTER(ConvDesc)]),
    "fc_conv_odd_path": (ct.c_int, [ct.POINTER(ConvDesc), ct.c_int, ct.POINTER(ct.c_int),
                                    ct.POINTER(ct.c_int), ct.POINTER(ct.c_int)]),
    "fc_edge_conv_odd": (ct.c_int, [ct.POINTER(ConvDesc), ct.c_int, ct.c_int,
                                    _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fc_edge_conv_odd_vjp": (ct.c_int, [ct.POINTER(ConvDesc), ct.c_int, ct.c_int,
                                        _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fc_scalar_readout": (ct.c_int, [ct.c_int, ct.c_int, ct.c_int, _vp, _vp, _vp, _vp]),
    "fc_edge_forces": (ct.c_int, [ct.c_int, ct.c_int, _vp, _vp, _vp, _vp]),
    "fc_ladder_num_paths": (ct.c_int, [ct.POINTER(LadderDesc)]),
    "fc_product_ladder_workspace_size": (ct.c_size_t, [ct.POINTER(LadderDesc), ct.c_int]),
    "fc_product_ladder": (ct.c_int, [ct.POINTER(LadderDesc), ct.c_int, _vp, _vp, _vp, _vp,
                                     _vp, _vp, ct.c_size_t, _vp]),
    "fc_product_ladder_vjp_workspace_size": (ct.c_size_t, [ct.POINTER(LadderDesc), ct.c_int]),
    "fc_product_ladder_vjp": (ct.c_int, [ct.POINTER(LadderDesc), ct.c_int, _vp, _vp, _vp, _vp,
                                         _vp, _vp, _vp, _vp, _vp, ct.c_size_t, _vp]),
    "fc_device_error": (ct.c_int, [ct.POINTER(ct.c_int), _vp]),
    "fc_set_wait_timeout": (ct.c_int, [ct.c_uint64]),
    "fc_edge_conv_workspace_size": (ct.c_size_t, [ct.POINTER(ConvDesc), ct.c_int, ct.c_int]),
    "fc_edge_conv_vjp_vjp": (ct.c_int, [ct.POINTER(ConvDesc), ct.c_int, ct.c_int] + [_vp] * 14),
    "fc_full_ladder_workspace_size": (ct.c_size_t, [ct.POINTER(LadderDesc), ct.c_int]),
    "fc_full_ladder": (ct.c_int, [ct.POINTER(LadderDesc), ct.c_int, _vp, _vp, _vp, _vp, _vp, _vp,
                                  ct.c_size_t, _vp]),
    "fc_full_ladder_vjp_workspace_size": (ct.c_size_t, [ct.POINTER(LadderDesc), ct.c_int]),
    "fc_full_ladder_vjp": (ct.c_int, [ct.POINTER(LadderDesc), ct.c_int] + [_vp] * 9
                           + [ct.c_size_t, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def lib():
    return _lib


def _check(status, where):
    if status != FC_OK:
        raise FlashCartError(status, where)


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return _vp(stream.cuda_stream)


def _ptr(t):
    return _vp(t.data_ptr()) if t is not None else None


def _dev(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t


def conv_desc(lmax, channels, sum_paths=False, envelope=None):
    """envelope: None, or (r_cut, edge_scale) for the cosine radial envelope."""
    if envelope is None:
        return ConvDesc(lmax, lmax, lmax, channels, int(bool(sum_paths)), 0, 0.0, 0.0)
    r_cut, scale = envelope
    return ConvDesc(lmax, lmax, lmax, channels, int(bool(sum_paths)), 1, float(r_cut),
                    float(scale))


def num_paths(lmax, channels=4, sum_paths=False):
    d = conv_desc(lmax, channels, sum_paths)
    n = _lib.fc_conv_num_paths(ct.byref(d))
    if n < 0:
        raise FlashCartError(4, "fc_conv_num_paths")
    return n


def out_row(lmax, channels=4, sum_paths=False):
    d = conv_desc(lmax, channels, sum_paths)
    n = _lib.fc_conv_out_row(ct.byref(d))
    if n < 0:
        raise FlashCartError(4, "fc_conv_out_row")
    return n


def paths(lmax):
    d = conv_desc(lmax, 4)
    out = []
    for p in range(num_paths(lmax)):
        a, b, c = ct.c_int(), ct.c_int(), ct.c_int()
        _check(_lib.fc_conv_path(ct.byref(d), p, ct.byref(a), ct.byref(b), ct.byref(c)),
               "fc_conv_path")
        out.append((a.value, b.value, c.value))
    return out


def odd_num_paths(lmax, channels=4, sum_paths=False):
    """Number of odd-J (Levi-Civita) paths at this rank."""
    d = conv_desc(lmax, channels, sum_paths)
    n = _lib.fc_conv_odd_num_paths(ct.byref(d))
    if n < 0:
        raise FlashCartError(4, "fc_conv_odd_num_paths")
    return n


def odd_out_row(lmax, channels=4, sum_paths=False):
    d = conv_desc(lmax, channels, sum_paths)
    n = _lib.fc_conv_odd_out_row(ct.byref(d))
    if n < 0:
        raise FlashCartError(4, "fc_conv_odd_out_row")
    return n


def odd_paths(lmax):
    d = conv_desc(lmax, 4)
    out = []
    for p in range(odd_num_paths(lmax)):
        a, b, c = ct.c_int(), ct.c_int(), ct.c_int()
        _check(_lib.fc_conv_odd_path(ct.byref(d), p, ct.byref(a), ct.byref(b), ct.byref(c)),
               "fc_conv_odd_path")
        out.append((a.value, b.value, c.value))
    return out


def build_rowptr(edge_index, edge_vec, n_nodes, stream=None, n_send=None):
    """Receiver row pointer [n_nodes+1] of a receiver-sorted edge list; raises
    FlashCartError(FC_ERR_CSR / FC_ERR_DEGENERATE_EDGE) on a bad graph.
    n_send: sender count when it differs from the receiver count (a
    receiver range of a larger graph)."""
    _dev(edge_index, torch.int32, "edge_index")
    E = edge_index.shape[1]
    if edge_vec is not None:
        _dev(edge_vec, torch.float32, "edge_vec")
        assert edge_vec.shape == (E, 3)
    dev = edge_index.device
    rowptr = torch.empty(n_nodes + 1, dtype=torch.int32, device=dev)
    flag = torch.empty(1, dtype=torch.int32, device=dev)
    _check(_lib.fc_build_rowptr_rect(n_nodes, n_nodes if n_send is None else n_send, E,
                                     _ptr(edge_index), _ptr(edge_vec), _ptr(rowptr), _ptr(flag),
                                     _stream(stream)), "fc_build_rowptr")
    return rowptr


def edge_conv(lmax, rowptr, edge_index, edge_vec, x, w, sum_paths=False,
              out=None, stream=None, envelope=None, odd=False):
    """z of Sec. 4 Eq. (1): [N][out_row * C].  odd=True: over the odd-J
    (Levi-Civita) paths (fc_edge_conv_odd; senders = receivers)."""
    _dev(rowptr, torch.int32, "rowptr")
    _dev(edge_index, torch.int32, "edge_index")
    _dev(edge_vec, torch.float32, "edge_vec")
    _dev(x, torch.float32, "x")
    _dev(w, torch.float32, "w")
    N = rowptr.shape[0] - 1
    E = edge_index.shape[1]
    C = x.shape[1] // ((lmax + 1) ** 2)
    d = conv_desc(lmax, C, sum_paths, envelope)
    zr = odd_out_row(lmax, C, sum_paths) if odd else out_row(lmax, C, sum_paths)
    NS = x.shape[0]     # senders: N, or all nodes of the graph for a receiver range
    if x.dim() != 2 or x.shape[1] != (lmax + 1) ** 2 * C:
        raise ValueError("x shape %s" % (tuple(x.shape),))
    if w.numel() != E * (odd_num_paths(lmax) if odd else num_paths(lmax)) * C:
        raise ValueError("w shape %s" % (tuple(w.shape),))
    if out is None:
        out = torch.empty((N, zr * C), dtype=torch.float32, device=x.device)
    else:
        _dev(out, torch.float32, "out")
        assert out.shape == (N, zr * C)
    if odd:
        if NS != N:
            raise ValueError("the odd-J convolution takes senders = receivers")
        _check(_lib.fc_edge_conv_odd(ct.byref(d), N, E, _ptr(rowptr), _ptr(edge_index),
                                     _ptr(edge_vec), _ptr(x), _ptr(w), _ptr(out),
                                     _stream(stream)), "fc_edge_conv_odd")
        return out
    _check(_lib.fc_edge_conv_rect(ct.byref(d), N, NS, E, _ptr(rowptr), _ptr(edge_index),
                                  _ptr(edge_vec), _ptr(x), _ptr(w), _ptr(out),
                                  _stream(stream)), "fc_edge_conv")
    return out


def edge_conv_vjp(lmax, rowptr, edge_index, edge_vec, x, w, g, sum_paths=False,
                  want=("x", "w", "r"), out=None, stream=None, envelope=None, odd=False):
    """(x_bar, w_bar, r_bar) of App. C Eq. (C1); entries not in `want` are None.
    odd=True: the VJP of the odd-J path convolution."""
    _dev(rowptr, torch.int32, "rowptr")
    _dev(edge_index, torch.int32, "edge_index")
    _dev(edge_vec, torch.float32, "edge_vec")
    _dev(x, torch.float32, "x")
    _dev(w, torch.float32, "w")
    _dev(g, torch.float32, "g")
    N = rowptr.shape[0] - 1
    E = edge_index.shape[1]
    C = x.shape[1] // ((lmax + 1) ** 2)
    d = conv_desc(lmax, C, sum_paths, envelope)
    P = odd_num_paths(lmax) if odd else num_paths(lmax)
    zr = odd_out_row(lmax, C, sum_paths) if odd else out_row(lmax, C, sum_paths)
    if g.shape != (N, zr * C):
        raise ValueError("g shape %s" % (tuple(g.shape),))
    if out is None:
        out = {}
    xb = out.get("x") if "x" in want else None
    wb = out.get("w") if "w" in want else None
    rb = out.get("r") if "r" in want else None
    if "x" in want and xb is None:
        xb = torch.empty_like(x)
    if "w" in want and wb is None:
        wb = torch.empty((E, P, C), dtype=torch.float32, device=x.device)
    if "r" in want and rb is None:
        rb = torch.empty((E, 3), dtype=torch.float32, device=x.device)
    if odd:
        _check(_lib.fc_edge_conv_odd_vjp(ct.byref(d), N, E, _ptr(rowptr), _ptr(edge_index),
                                         _ptr(edge_vec), _ptr(x), _ptr(w), _ptr(g), _ptr(xb),
                                         _ptr(wb), _ptr(rb), _stream(stream)), "fc_edge_conv_odd_vjp")
        return xb, wb, rb
    _check(_lib.fc_edge_conv_vjp_rect(ct.byref(d), N, x.shape[0], E, _ptr(rowptr), _ptr(edge_index),
                                      _ptr(edge_vec), _ptr(x), _ptr(w), _ptr(g), _ptr(xb),
                                      _ptr(wb), _ptr(rb), _stream(stream)), "fc_edge_conv_vjp")
    return xb, wb, rb


def edge_conv_vjp_vjp(lmax, rowptr, edge_index, edge_vec, x, w, g, v_x=None, v_w=None,
                      v_r=None, sum_paths=False, want=("g", "x", "w", "r"), stream=None):
    """(g_hat, x_hat, w_hat, r_hat) of App. C Eq. C2 (Algorithm 3): the
    gradients of <v_x, x_bar> + <v_w, w_bar> + <v_r, r_bar> with respect to
    g, x, w and the edge vectors; None cotangents are zero, outputs not in
    `want` are None."""
    for t, n in ((x, "x"), (g, "g")):
        _dev(t, torch.float32, n)
    _dev(rowptr, torch.int32, "rowptr")
    _dev(edge_index, torch.int32, "edge_index")
    for t, n in ((v_x, "v_x"), (v_w, "v_w"), (v_r, "v_r")):
        if t is not None:
            _dev(t, torch.float32, n)
    N = rowptr.shape[0] - 1
    E = edge_index.shape[1]
    C = x.shape[1] // ((lmax + 1) ** 2)
    d = conv_desc(lmax, C, sum_paths)
    P = num_paths(lmax)
    if g.shape != (N, out_row(lmax, C, sum_paths) * C):
        raise ValueError("g shape %s" % (tuple(g.shape),))
    gh = torch.empty_like(g) if "g" in want else None
    xh = torch.empty_like(x) if "x" in want else None
    wh = torch.empty((E, P, C), dtype=torch.float32, device=x.device) if "w" in want else None
    rh = torch.empty((E, 3), dtype=torch.float32, device=x.device) if "r" in want else None
    _check(_lib.fc_edge_conv_vjp_vjp(ct.byref(d), N, E, _ptr(rowptr), _ptr(edge_index),
                                     _ptr(edge_vec), _ptr(x), _ptr(w), _ptr(g), _ptr(v_x),
                                     _ptr(v_w), _ptr(v_r), _ptr(gh), _ptr(xh), _ptr(wh),
                                     _ptr(rh), _stream(stream)), "fc_edge_conv_vjp_vjp")
    return gh, xh, wh, rh


def _workspace(nbytes, device):
    if nbytes == 0:
        return None
    return torch.empty((nbytes + 15) // 16 * 4, dtype=torch.float32, device=device)


def _scratch(workspace, need, device):
    """(buffer, its size in bytes): a new buffer of `need` bytes, or the
    caller's tensor with its actual size, which the library checks."""
    if workspace is None:
        return _workspace(need, device), need
    if not (workspace.is_cuda and workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return workspace, workspace.numel() * workspace.element_size()


def ladder_workspace_bytes(lmax, channels, order, n_nodes, vjp=False):
    """Scratch bytes fc_product_ladder (or, with vjp=True, its VJP) needs."""
    d = LadderDesc(lmax, channels, order)
    f = _lib.fc_product_ladder_vjp_workspace_size if vjp else _lib.fc_product_ladder_workspace_size
    return f(ct.byref(d), n_nodes)


def product_ladder(lmax, order, A1, path_w, mix_w, workspace=None, stream=None):
    """(states [order-1][N][...], z) of Sec. 5 Eq. (2), path-reduced products
    followed by a per-rank channel mix."""
    _dev(A1, torch.float32, "A1")
    N = A1.shape[0]
    NY = (lmax + 1) ** 2
    C = A1.shape[1] // NY
    d = LadderDesc(lmax, C, order)
    S = order - 1
    states = torch.empty((max(S, 0), N, NY * C), dtype=torch.float32, device=A1.device)
    z = torch.empty_like(A1)
    ws_bytes = _lib.fc_product_ladder_workspace_size(ct.byref(d), N)
    workspace, ws_bytes = _scratch(workspace, ws_bytes, A1.device)
    if S > 0:
        _dev(path_w, torch.float32, "path_w")
        _dev(mix_w, torch.float32, "mix_w")
    _check(_lib.fc_product_ladder(ct.byref(d), N, _ptr(A1), _ptr(path_w) if S > 0 else None,
                                  _ptr(mix_w) if S > 0 else None, _ptr(states) if S > 0 else None,
                                  _ptr(z), _ptr(workspace), ws_bytes if workspace is not None else 0,
                                  _stream(stream)), "fc_product_ladder")
    return states, z


def product_ladder_vjp(lmax, order, A1, path_w, mix_w, states, gz, workspace=None,
                       stream=None):
    """(A1_bar, path_w_bar, mix_w_bar) of fc_product_ladder."""
    _dev(A1, torch.float32, "A1")
    _dev(gz, torch.float32, "gz")
    N = A1.shape[0]
    NY = (lmax + 1) ** 2
    C = A1.shape[1] // NY
    d = LadderDesc(lmax, C, order)
    S = order - 1
    A1b = torch.empty_like(A1)
    pwb = torch.empty((max(S, 0),) + tuple(path_w.shape[1:]), dtype=torch.float32, device=A1.device)
    mwb = torch.empty((max(S, 0),) + tuple(mix_w.shape[1:]), dtype=torch.float32, device=A1.device)
    ws_bytes = _lib.fc_product_ladder_vjp_workspace_size(ct.byref(d), N)
    workspace, ws_bytes = _scratch(workspace, ws_bytes, A1.device)
    _check(_lib.fc_product_ladder_vjp(
        ct.byref(d), N, _ptr(A1), _ptr(path_w) if S > 0 else None,
        _ptr(mix_w) if S > 0 else None, _ptr(states) if S > 0 else None, _ptr(gz),
        _ptr(A1b), _ptr(pwb) if S > 0 else None, _ptr(mwb) if S > 0 else None,
        _ptr(workspace), ws_bytes if workspace is not None else 0, _stream(stream)),
        "fc_product_ladder_vjp")
    return A1b, pwb, mwb


def full_ladder(lmax, order, A, W1, Wq, workspace=None, stream=None):
    """(states [order][N][...] = phi_1..phi_order, z) of the full ladder
    (Sec. 5 Eq. 2): path-separated products, per-rank path+channel maps."""
    _dev(A, torch.float32, "A")
    _dev(W1, torch.float32, "W1")
    N = A.shape[0]
    NY = (lmax + 1) ** 2
    C = A.shape[1] // NY
    d = LadderDesc(lmax, C, order)
    states = torch.empty((order, N, NY * C), dtype=torch.float32, device=A.device)
    z = torch.empty_like(A)
    if order > 1:
        _dev(Wq, torch.float32, "Wq")
    ws_bytes = _lib.fc_full_ladder_workspace_size(ct.byref(d), N)
    workspace, ws_bytes = _scratch(workspace, ws_bytes, A.device)
    _check(_lib.fc_full_ladder(ct.byref(d), N, _ptr(A), _ptr(W1), _ptr(Wq) if order > 1 else None,
                               _ptr(states), _ptr(z), _ptr(workspace),
                               ws_bytes if workspace is not None else 0, _stream(stream)),
           "fc_full_ladder")
    return states, z


def full_ladder_vjp(lmax, order, A, W1, Wq, states, gz, workspace=None, stream=None):
    """(A_bar, W1_bar, Wq_bar): gradients of <gz, z> for fc_full_ladder,
    given the states phi_1..phi_order it returned."""
    for t, n in ((A, "A"), (W1, "W1"), (states, "states"), (gz, "gz")):
        _dev(t, torch.float32, n)
    N = A.shape[0]
    NY = (lmax + 1) ** 2
    C = A.shape[1] // NY
    d = LadderDesc(lmax, C, order)
    Ab = torch.empty_like(A)
    W1b = torch.empty_like(W1)
    if order > 1:
        _dev(Wq, torch.float32, "Wq")
        Wqb = torch.empty_like(Wq)
    else:
        Wqb = None
    ws_bytes = _lib.fc_full_ladder_vjp_workspace_size(ct.byref(d), N)
    workspace, ws_bytes = _scratch(workspace, ws_bytes, A.device)
    _check(_lib.fc_full_ladder_vjp(ct.byref(d), N, _ptr(A), _ptr(W1), _ptr(Wq) if order > 1 else None,
                                   _ptr(states), _ptr(gz), _ptr(Ab), _ptr(W1b), _ptr(Wqb),
                                   _ptr(workspace), ws_bytes if workspace is not None else 0,
                                   _stream(stream)), "fc_full_ladder_vjp")
    return Ab, W1b, Wqb


def device_error(stream=None):
    """Sticky error word of the kernels with bounded barrier waits (0 = none
    gave up since the last call); synchronises the stream and clears it."""
    flag = ct.c_int(0)
    _check(_lib.fc_device_error(ct.byref(flag), _stream(stream)), "fc_device_error")
    return flag.value


def set_wait_timeout(ns=0):
    """Bound (ns) of the tensor-core kernels' barrier waits on the current
    device; 0 restores the default."""
    _check(_lib.fc_set_wait_timeout(int(ns)), "fc_set_wait_timeout")


def scalar_readout(lmax, z, want_grad=True, stream=None):
    """(energy [1], gz) with energy = sum of the rank-0 block of z and
    gz = d energy / d z."""
    _dev(z, torch.float32, "z")
    N = z.shape[0]
    C = z.shape[1] // ((lmax + 1) ** 2)
    energy = torch.empty(1, dtype=torch.float32, device=z.device)
    gz = torch.empty_like(z) if want_grad else None
    _check(_lib.fc_scalar_readout(N, lmax, C, _ptr(z), _ptr(energy), _ptr(gz),
                                  _stream(stream)), "fc_scalar_readout")
    return energy, gz


def edge_forces(edge_index, r_bar, n_nodes, stream=None):
    """forces [N][3] = -dE/dpos from per-edge gradients r_bar."""
    _dev(edge_index, torch.int32, "edge_index")
    _dev(r_bar, torch.float32, "r_bar")
    F = torch.empty((n_nodes, 3), dtype=torch.float32, device=r_bar.device)
    _check(_lib.fc_edge_forces(n_nodes, edge_index.shape[1], _ptr(edge_index), _ptr(r_bar),
                               _ptr(F), _stream(stream)), "fc_edge_forces")
    return F


def interaction_block(lmax, order, rowptr, edge_index, edge_vec, x, omega, path_w, mix_w,
                      r_cut, edge_scale, stream=None):
    """Energy and forces of one interaction block, each step a library call:
    edge convolution with paths summed per output rank and the cosine
    envelope (App. E Eq. E1 with the 1/sqrt(mean neighbours) factor in
    edge_scale), the product ladder (Sec. 5 Eq. 2), E = sum of its rank-0
    outputs, then the ladder VJP, the convolution VJP (r_bar only) and the
    force scatter.  Returns (energy [1], forces [N][3], z)."""
    env = (r_cut, edge_scale)
    N = rowptr.shape[0] - 1
    A1 = edge_conv(lmax, rowptr, edge_index, edge_vec, x, omega, sum_paths=True,
                   envelope=env, stream=stream)
    states, z = product_ladder(lmax, order, A1, path_w, mix_w, stream=stream)
    energy, gz = scalar_readout(lmax, z, stream=stream)
    A1b, _, _ = product_ladder_vjp(lmax, order, A1, path_w, mix_w, states, gz, stream=stream)
    _, _, rb = edge_conv_vjp(lmax, rowptr, edge_index, edge_vec, x, omega, A1b, sum_paths=True,
                             want=("r",), envelope=env, stream=stream)
    F = edge_forces(edge_index, rb, N, stream=stream)
    return energy, F, z
