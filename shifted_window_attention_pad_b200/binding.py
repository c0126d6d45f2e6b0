"""Python binding of libswinwattn.so: argument marshalling only.

Same names as the C ABI in include/swin_wattn.h. Every step of the
computation runs in the library's CUDA kernels; this module checks tensor
devices, dtypes and contiguity, passes raw pointers and the current CUDA
stream, and turns negative status codes into exceptions. torch is used for
device memory and streams only. There is no fallback: if the library is
missing, the first call raises.
"""
import ctypes
import os

import torch

from .workloads import Workload

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libswinwattn.so")

SWIN_OK = 0
SWIN_ERR_TIMEOUT = -5
SWIN_DTYPE_F32 = 0
SWIN_DTYPE_BF16 = 1
SWIN_FLAG_FORCE_GENERIC = 1
SWIN_FLAG_TEST_TIMEOUT = 2
SWIN_FLAG_FORCE_TILED = 4
SWIN_FLAG_DBIAS_SUMS = 8

EXPORTED = ("swin_wattn_path", "swin_wattn_workspace_size", "swin_wattn_fwd", "swin_wattn_bwd",
            "swin_wattn_bwd_noalloc", "swin_wattn_index_map", "swin_wattn_layout_map",
            "swin_wattn_dbias_sums", "swin_wattn_dbias_finish", "swin_wattn_fwd_band",
            "swin_wattn_bwd_band", "swin_wattn_poll_status",
            "swin_wattn_strerror", "swin_wattn_launch_count")
SWIN_NOALLOC_SCRATCH_BYTES = 1 << 20   # include/swin_wattn.h


class SwinWattnDesc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "H", "W", "win_h", "win_w", "shift_h", "shift_w", "heads", "head_dim",
                 "dtype", "flags", "valid_h", "valid_w")]


class SwinWattnHalo(ctypes.Structure):
    """Halo rows of a row band (include/swin_wattn.h): inputs below the band
    and the outputs that belong to the next band."""
    _fields_ = [("interior", ctypes.c_int32), ("q", ctypes.c_void_p), ("k", ctypes.c_void_p),
                ("v", ctypes.c_void_p), ("dout", ctypes.c_void_p), ("out", ctypes.c_void_p),
                ("lse", ctypes.c_void_p), ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p),
                ("dv", ctypes.c_void_p)]


class SwinWattnError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__("%s: status %d (%s)" % (what, status, swin_wattn_strerror(status)))


_lib = None


def lib():
    """Load libswinwattn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libswinwattn.so not built: run __graft_entry__.build() "
                              "(or python shifted_window_attention_pad_b200/build.py)")
        L = ctypes.CDLL(LIB_PATH)
        D = ctypes.POINTER(SwinWattnDesc)
        P = ctypes.c_void_p
        L.swin_wattn_path.argtypes = [D]
        L.swin_wattn_workspace_size.argtypes = [D, ctypes.POINTER(ctypes.c_size_t)]
        L.swin_wattn_fwd.argtypes = [D, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.swin_wattn_bwd.argtypes = [D, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.swin_wattn_bwd_noalloc.argtypes = [D, P, P, P, P, P, P, P, P, P, P]
        L.swin_wattn_index_map.argtypes = [D, P, P]
        L.swin_wattn_layout_map.argtypes = [D, P, P, P, P]
        L.swin_wattn_dbias_sums.argtypes = [D, ctypes.POINTER(ctypes.c_size_t),
                                            ctypes.POINTER(ctypes.c_size_t)]
        L.swin_wattn_dbias_finish.argtypes = [D, P, P, P]
        HP = ctypes.POINTER(SwinWattnHalo)
        L.swin_wattn_fwd_band.argtypes = [D, HP, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.swin_wattn_bwd_band.argtypes = [D, HP, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.swin_wattn_poll_status.argtypes = [P, ctypes.POINTER(ctypes.c_int), P]
        L.swin_wattn_strerror.argtypes = [ctypes.c_int]
        L.swin_wattn_strerror.restype = ctypes.c_char_p
        L.swin_wattn_launch_count.argtypes = []
        L.swin_wattn_launch_count.restype = ctypes.c_uint64
        for f in ("swin_wattn_path", "swin_wattn_workspace_size", "swin_wattn_fwd",
                  "swin_wattn_bwd", "swin_wattn_bwd_noalloc", "swin_wattn_index_map",
                  "swin_wattn_layout_map", "swin_wattn_dbias_sums", "swin_wattn_dbias_finish",
                  "swin_wattn_fwd_band", "swin_wattn_bwd_band", "swin_wattn_poll_status"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def make_desc(B, H, W, win, shift, heads, head_dim, dtype, flags=0, valid=None):
    """`valid` = (valid_h, valid_w), the extent of tokens that carry field data
    (None: the whole grid)."""
    wh, ww = (win, win) if isinstance(win, int) else win
    sh, sw = (shift, shift) if isinstance(shift, int) else shift
    dt = SWIN_DTYPE_BF16 if dtype in ("bf16", torch.bfloat16, SWIN_DTYPE_BF16) else SWIN_DTYPE_F32
    vh, vw = valid if valid is not None else (0, 0)
    return SwinWattnDesc(B, H, W, wh, ww, sh, sw, heads, head_dim, dt, flags, vh, vw)


def field_valid_extent(field_h, field_w, patch):
    """Valid token extent of a field of field_h x field_w real pixels cut into
    patch x patch tokens: a token is real when its patch holds a real pixel."""
    return -(-field_h // patch), -(-field_w // patch)


def desc_for(wl: Workload, flags=0):
    return make_desc(wl.B, wl.H, wl.W, wl.win, wl.shift, wl.heads, wl.head_dim, wl.dtype, flags,
                     wl.valid)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t, dtype=None, name="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    return ctypes.c_void_p(t.data_ptr())


def _check(rc, what):
    if rc != SWIN_OK:
        raise SwinWattnError(rc, what)


def _elem(desc):
    return torch.bfloat16 if desc.dtype == SWIN_DTYPE_BF16 else torch.float32


def swin_wattn_strerror(status):
    return lib().swin_wattn_strerror(status).decode()


def swin_wattn_path(desc):
    rc = lib().swin_wattn_path(ctypes.byref(desc))
    if rc < 0:
        raise SwinWattnError(rc, "swin_wattn_path")
    return rc


def swin_wattn_workspace_size(desc):
    n = ctypes.c_size_t(0)
    _check(lib().swin_wattn_workspace_size(ctypes.byref(desc), ctypes.byref(n)),
           "swin_wattn_workspace_size")
    return n.value


def new_workspace(desc, device="cuda"):
    """Caller-owned workspace of the size the library asks for (zeroed once)."""
    return torch.zeros(swin_wattn_workspace_size(desc), dtype=torch.uint8, device=device)


def swin_wattn_fwd(desc, q, k, v, bias_table, out, lse=None, workspace=None, stream=None):
    el = _elem(desc)
    if workspace is None:
        workspace = new_workspace(desc, q.device)
    rc = lib().swin_wattn_fwd(ctypes.byref(desc), _ptr(q, el, "q"), _ptr(k, el, "k"),
                              _ptr(v, el, "v"), _ptr(bias_table, torch.float32, "bias_table"),
                              _ptr(out, el, "out"), _ptr(lse, torch.float32, "lse"),
                              _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                              _stream(stream))
    _check(rc, "swin_wattn_fwd")
    return out


def swin_wattn_bwd(desc, q, k, v, bias_table, dout, dq, dk, dv, dbias_table, workspace=None,
                   stream=None):
    el = _elem(desc)
    if workspace is None:
        workspace = new_workspace(desc, q.device)
    rc = lib().swin_wattn_bwd(ctypes.byref(desc), _ptr(q, el, "q"), _ptr(k, el, "k"),
                              _ptr(v, el, "v"), _ptr(bias_table, torch.float32, "bias_table"),
                              _ptr(dout, el, "dout"), _ptr(dq, el, "dq"), _ptr(dk, el, "dk"),
                              _ptr(dv, el, "dv"), _ptr(dbias_table, torch.float32, "dbias_table"),
                              _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                              _stream(stream))
    _check(rc, "swin_wattn_bwd")
    return dq, dk, dv, dbias_table


def make_halo(interior, q=None, k=None, v=None, dout=None, out=None, lse=None, dq=None, dk=None,
              dv=None):
    """SwinWattnHalo from device tensors ([B, shift_h, W, heads, head_dim])."""
    p = lambda t, n: _ptr(t, None, n) if t is not None else None
    return SwinWattnHalo(int(interior), p(q, "halo q"), p(k, "halo k"), p(v, "halo v"),
                         p(dout, "halo dout"), p(out, "halo out"), p(lse, "halo lse"),
                         p(dq, "halo dq"), p(dk, "halo dk"), p(dv, "halo dv"))


def swin_wattn_fwd_band(desc, halo, q, k, v, bias_table, out, lse=None, workspace=None,
                        stream=None):
    el = _elem(desc)
    if workspace is None:
        workspace = new_workspace(desc, q.device)
    rc = lib().swin_wattn_fwd_band(ctypes.byref(desc), ctypes.byref(halo), _ptr(q, el, "q"),
                                   _ptr(k, el, "k"), _ptr(v, el, "v"),
                                   _ptr(bias_table, torch.float32, "bias_table"),
                                   _ptr(out, el, "out"), _ptr(lse, torch.float32, "lse"),
                                   _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                                   _stream(stream))
    _check(rc, "swin_wattn_fwd_band")
    return out


def swin_wattn_bwd_band(desc, halo, q, k, v, bias_table, dout, dq, dk, dv, dbias_table,
                        workspace=None, stream=None):
    el = _elem(desc)
    if workspace is None:
        workspace = new_workspace(desc, q.device)
    rc = lib().swin_wattn_bwd_band(ctypes.byref(desc), ctypes.byref(halo), _ptr(q, el, "q"),
                                   _ptr(k, el, "k"), _ptr(v, el, "v"),
                                   _ptr(bias_table, torch.float32, "bias_table"),
                                   _ptr(dout, el, "dout"), _ptr(dq, el, "dq"), _ptr(dk, el, "dk"),
                                   _ptr(dv, el, "dv"),
                                   _ptr(dbias_table, torch.float32, "dbias_table"),
                                   _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                                   _stream(stream))
    _check(rc, "swin_wattn_bwd_band")
    return dq, dk, dv, dbias_table


def swin_wattn_bwd_noalloc(desc, q, k, v, bias_table, dout, dq, dk, dv, dbias_table,
                           stream=None):
    """swin_wattn_bwd with the library's static scratch instead of a workspace
    (for callers that cannot allocate; see include/swin_wattn.h)."""
    el = _elem(desc)
    rc = lib().swin_wattn_bwd_noalloc(ctypes.byref(desc), _ptr(q, el, "q"), _ptr(k, el, "k"),
                                      _ptr(v, el, "v"),
                                      _ptr(bias_table, torch.float32, "bias_table"),
                                      _ptr(dout, el, "dout"), _ptr(dq, el, "dq"),
                                      _ptr(dk, el, "dk"), _ptr(dv, el, "dv"),
                                      _ptr(dbias_table, torch.float32, "dbias_table"),
                                      _stream(stream))
    _check(rc, "swin_wattn_bwd_noalloc")
    return dq, dk, dv, dbias_table


def swin_wattn_index_map(desc, out=None, stream=None):
    if out is None:
        Hp = -(-desc.H // desc.win_h) * desc.win_h
        Wp = -(-desc.W // desc.win_w) * desc.win_w
        out = torch.empty((desc.B, Hp // desc.win_h, Wp // desc.win_w, desc.win_h * desc.win_w),
                          dtype=torch.int32, device="cuda")
    _check(lib().swin_wattn_index_map(ctypes.byref(desc), _ptr(out, torch.int32, "map"),
                                      _stream(stream)), "swin_wattn_index_map")
    return out


def swin_wattn_dbias_sums(desc):
    """(offset, bytes) of the exact bias-gradient sums in the workspace."""
    off, n = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(lib().swin_wattn_dbias_sums(ctypes.byref(desc), ctypes.byref(off), ctypes.byref(n)),
           "swin_wattn_dbias_sums")
    return off.value, n.value


def dbias_sums_view(desc, workspace):
    """The exact sums inside `workspace` as an int64 tensor (a view, no copy)."""
    off, n = swin_wattn_dbias_sums(desc)
    return workspace[off:off + n].view(torch.int64)


def swin_wattn_dbias_finish(desc, workspace, dbias_table, stream=None):
    _check(lib().swin_wattn_dbias_finish(ctypes.byref(desc),
                                         _ptr(workspace, torch.uint8, "workspace"),
                                         _ptr(dbias_table, torch.float32, "dbias_table"),
                                         _stream(stream)), "swin_wattn_dbias_finish")
    return dbias_table


def swin_wattn_layout_map(desc, stream=None):
    """(map, labels) of the tcgen05 kernels' own layout stage, both int32
    [B, H^/win_h, W^/win_w, win_h*win_w] on the device."""
    Hp = -(-desc.H // desc.win_h) * desc.win_h
    Wp = -(-desc.W // desc.win_w) * desc.win_w
    shape = (desc.B, Hp // desc.win_h, Wp // desc.win_w, desc.win_h * desc.win_w)
    ids = torch.empty(desc.B * desc.H * desc.W * desc.heads * desc.head_dim, dtype=torch.bfloat16,
                      device="cuda")
    m = torch.empty(shape, dtype=torch.int32, device="cuda")
    lab = torch.empty(shape, dtype=torch.int32, device="cuda")
    _check(lib().swin_wattn_layout_map(ctypes.byref(desc), _ptr(ids, torch.bfloat16, "ids"),
                                       _ptr(m, torch.int32, "map"), _ptr(lab, torch.int32, "labels"),
                                       _stream(stream)), "swin_wattn_layout_map")
    return m, lab


def swin_wattn_poll_status(workspace, stream=None):
    st = ctypes.c_int(0)
    _check(lib().swin_wattn_poll_status(_ptr(workspace, torch.uint8, "workspace"),
                                        ctypes.byref(st), _stream(stream)),
           "swin_wattn_poll_status")
    return st.value


def swin_wattn_launch_count():
    return int(lib().swin_wattn_launch_count())


# ---- convenience wrappers (allocate outputs with torch, then call the ABI) -------
def forward(desc, q, k, v, bias_table, want_lse=False, workspace=None):
    out = torch.empty_like(q)
    lse = (torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device) if want_lse else None)
    swin_wattn_fwd(desc, q, k, v, bias_table, out, lse, workspace)
    return (out, lse) if want_lse else out


def backward(desc, q, k, v, bias_table, dout, workspace=None):
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dT = torch.empty_like(bias_table)
    swin_wattn_bwd(desc, q, k, v, bias_table, dout, dq, dk, dv, dT, workspace)
    return dq, dk, dv, dT
