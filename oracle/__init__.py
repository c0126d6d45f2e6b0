"""fp64 CPU oracle for shifted-window multi-head self-attention over a padded grid.

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package. The product path (the
CUDA library and its Python binding) never imports it, and the two share no
code.

The arithmetic lives in ``swin_oracle.c`` (steps: pad, cyclic shift, window
partition, masked softmax attention with relative-position bias, window
reverse, reverse shift, crop; see that file's header for the page passages and
readings). This module only marshals numpy arrays through ctypes.
"""
import ctypes
import numpy as np

from . import build as _build


class Shape(ctypes.Structure):
    """Problem shape; valid_h / valid_w (0 = H / W) bound the tokens that carry
    field data (the others are padding, see swin_oracle.c)."""
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "H", "W", "win_h", "win_w", "shift_h", "shift_w", "heads", "head_dim",
                 "valid_h", "valid_w")]


_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        S = ctypes.POINTER(Shape)
        L.swin_oracle_forward.argtypes = [S, P, P, P, P, P, P]
        L.swin_oracle_backward.argtypes = [S, P, P, P, P, P, P, P, P, P]
        L.swin_oracle_index_map.argtypes = [S, P]
        L.swin_oracle_region_labels.argtypes = [S, P]
        L.swin_oracle_roundtrip.argtypes = [S, P, P, ctypes.c_int]
        for f in ("swin_oracle_forward", "swin_oracle_backward", "swin_oracle_index_map",
                  "swin_oracle_region_labels", "swin_oracle_roundtrip", "swin_oracle_num_threads"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def num_threads() -> int:
    return lib().swin_oracle_num_threads()


def make_shape(B, H, W, win, shift, heads, head_dim, valid=None):
    wh, ww = (win, win) if np.isscalar(win) else win
    sh, sw = (shift, shift) if np.isscalar(shift) else shift
    vh, vw = valid if valid is not None else (0, 0)
    return Shape(B, H, W, wh, ww, sh, sw, heads, head_dim, vh, vw)


def padded_hw(s: Shape):
    return (-(-s.H // s.win_h) * s.win_h, -(-s.W // s.win_w) * s.win_w)


def n_bins(s: Shape) -> int:
    return (2 * s.win_h - 1) * (2 * s.win_w - 1)


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError("%s failed with status %d" % (what, rc))


def forward(s: Shape, q, k, v, table, want_lse=True):
    """Returns (out fp64 [B,H,W,heads,hd], lse fp64 [B,H,W,heads] or None)."""
    q, k, v, T = _f64(q), _f64(k), _f64(v), _f64(table)
    grid = (s.B, s.H, s.W, s.heads, s.head_dim)
    for name, a in (("q", q), ("k", k), ("v", v)):
        assert a.shape == grid, (name, a.shape, grid)
    assert T.shape == (n_bins(s), s.heads), T.shape
    out = np.zeros(grid, np.float64)
    lse = np.zeros(grid[:4], np.float64) if want_lse else None
    rc = lib().swin_oracle_forward(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(T),
                                   _ptr(out), _ptr(lse) if want_lse else None)
    _check(rc, "swin_oracle_forward")
    return out, lse


def backward(s: Shape, q, k, v, table, dout):
    """Returns (dq, dk, dv, dtable), all fp64."""
    q, k, v, do, T = _f64(q), _f64(k), _f64(v), _f64(dout), _f64(table)
    grid = (s.B, s.H, s.W, s.heads, s.head_dim)
    dq, dk, dv = (np.zeros(grid, np.float64) for _ in range(3))
    dT = np.zeros((n_bins(s), s.heads), np.float64)
    rc = lib().swin_oracle_backward(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(T),
                                    _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dT))
    _check(rc, "swin_oracle_backward")
    return dq, dk, dv, dT


def index_map(s: Shape):
    """int64 [B, nWy*nWx, win_h*win_w]: source token (b*H+y)*W+x of each slot, -1 for pad."""
    Hp, Wp = padded_hw(s)
    m = np.empty((s.B, (Hp // s.win_h) * (Wp // s.win_w), s.win_h * s.win_w), np.int64)
    _check(lib().swin_oracle_index_map(ctypes.byref(s), _ptr(m)), "swin_oracle_index_map")
    return m


def region_labels(s: Shape):
    """int32 [nWy*nWx, win_h*win_w]: shift-mask region label of each slot."""
    Hp, Wp = padded_hw(s)
    lab = np.empty(((Hp // s.win_h) * (Wp // s.win_w), s.win_h * s.win_w), np.int32)
    _check(lib().swin_oracle_region_labels(ctypes.byref(s), _ptr(lab)), "swin_oracle_region_labels")
    return lab


def roundtrip(s: Shape, grid, which: str):
    """Apply partition->reverse ('partition') or roll->unroll ('roll') to an int64 H^xW^ grid."""
    g = np.ascontiguousarray(np.asarray(grid, np.int64))
    Hp, Wp = padded_hw(s)
    assert g.shape == (Hp, Wp)
    out = np.empty_like(g)
    rc = lib().swin_oracle_roundtrip(ctypes.byref(s), _ptr(g), _ptr(out),
                                     0 if which == "partition" else 1)
    _check(rc, "swin_oracle_roundtrip")
    return out
