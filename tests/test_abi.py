"""C-ABI checks that need no GPU: the library loads, exports every function that
include/swin_wattn.h declares, and rejects bad arguments on the host before any
CUDA call."""
import ctypes
import os
import re

import pytest

from shifted_window_attention_pad_b200 import WORKLOADS, binding as sb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(swin_\w+)\s*\(", text, flags=re.M)
    return names


@pytest.fixture(scope="module")
def L():
    from shifted_window_attention_pad_b200 import build
    build.build()
    return sb.lib()


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("swin_wattn_fwd", "swin_wattn_bwd", "swin_wattn_workspace_size",
              "swin_wattn_index_map", "swin_wattn_strerror"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for n in declared_functions():
        assert hasattr(L, n), n
        assert ctypes.cast(getattr(L, n), ctypes.c_void_p).value


def test_path_selection_on_the_workloads(L):
    """tcgen05 kernels for bf16 64-token windows (1) and 256-token windows (3),
    portable kernels (0) for fp32."""
    expect = {"tiny-16x16-w4": 0, "ragged-90x180-w8": 1, "twelfth-degree-256x544-w8": 1,
              "downsampled-128x272-w16": 3, "small-patch-2x512x1088-w8": 1}
    for name, want in expect.items():
        assert sb.swin_wattn_path(sb.desc_for(WORKLOADS[name])) == want, name
    d = sb.desc_for(WORKLOADS["twelfth-degree-256x544-w8"], flags=sb.SWIN_FLAG_FORCE_GENERIC)
    assert sb.swin_wattn_path(d) == 0
    d = sb.desc_for(WORKLOADS["twelfth-degree-256x544-w8"], flags=sb.SWIN_FLAG_FORCE_TILED)
    assert sb.swin_wattn_path(d) == 2
    d = sb.desc_for(WORKLOADS["downsampled-128x272-w16"], flags=sb.SWIN_FLAG_FORCE_TILED)
    assert sb.swin_wattn_path(d) == 2
    d = sb.desc_for(WORKLOADS["tiny-16x16-w4"], flags=sb.SWIN_FLAG_FORCE_TILED)
    assert sb.swin_wattn_path(d) == 0      # fp32 has no tensor-core path


@pytest.mark.parametrize("win,hd,want", [((7, 7), 64, 2), ((8, 12), 32, 2), ((16, 16), 64, 3),
                                         ((16, 16), 32, 3), ((8, 32), 64, 3), ((16, 8), 64, 2),
                                         ((12, 12), 32, 2), ((16, 17), 64, 0), ((32, 32), 64, 4),
                                         ((32, 32), 128, 4), ((32, 32), 32, 0),
                                         ((16, 16), 128, 0), ((8, 8), 64, 1), ((8, 8), 128, 1),
                                         ((4, 16), 128, 1), ((7, 7), 128, 0)])
def test_tensor_core_paths_cover_windows_up_to_1024_tokens(L, win, hd, want):
    d = sb.make_desc(1, 40, 52, win, (win[0] // 2, win[1] // 2), 2, hd, "bf16")
    assert sb.swin_wattn_path(d) == want


@pytest.mark.parametrize("shift,want", [((16, 16), 4), ((14, 16), 4), ((0, 0), 4), ((2, 12), 4),
                                        ((15, 16), 4), ((16, 6), 4), ((16, 3), 0), ((13, 5), 0)])
def test_1024_token_windows_need_sub_boxes_of_whole_swizzle_atoms(L, shift, want):
    """A 128-token block's sub-boxes (rows of 4, or the two parts at the row
    seam, times the column segments) must each hold a multiple of 8 rows."""
    d = sb.make_desc(1, 64, 96, (32, 32), shift, 2, 128, "bf16")
    assert sb.swin_wattn_path(d) == want


@pytest.mark.parametrize("field,value", [("shift_h", 8), ("shift_w", -1), ("win_h", 0),
                                         ("head_dim", 12), ("heads", 0), ("B", 0), ("H", 0),
                                         ("win_w", 65), ("head_dim", 264)])
def test_bad_descriptions_are_rejected_on_the_host(L, field, value):
    d = sb.desc_for(WORKLOADS["twelfth-degree-256x544-w8"])
    setattr(d, field, value)
    assert L.swin_wattn_path(ctypes.byref(d)) == -1
    n = ctypes.c_size_t(0)
    assert L.swin_wattn_workspace_size(ctypes.byref(d), ctypes.byref(n)) == -1


def test_bad_dtype_is_unsupported(L):
    d = sb.desc_for(WORKLOADS["tiny-16x16-w4"])
    d.dtype = 7
    assert L.swin_wattn_path(ctypes.byref(d)) == -2


def test_null_and_misaligned_pointers_are_rejected_before_any_cuda_call(L):
    d = sb.desc_for(WORKLOADS["ragged-90x180-w8"])
    P = ctypes.c_void_p
    good = P(1 << 20)
    assert L.swin_wattn_fwd(ctypes.byref(d), None, good, good, good, good, None, good, 1 << 30,
                            None) == -1
    assert L.swin_wattn_fwd(ctypes.byref(d), P((1 << 20) + 2), good, good, good, good, None,
                            good, 1 << 30, None) == -1
    assert L.swin_wattn_bwd(ctypes.byref(d), good, good, good, good, good, good, good, None,
                            good, good, 1 << 30, None) == -1
    # workspace: too small, misaligned
    assert L.swin_wattn_fwd(ctypes.byref(d), good, good, good, good, good, None, good, 16,
                            None) == -3
    assert L.swin_wattn_fwd(ctypes.byref(d), good, good, good, good, good, None, P((1 << 20) + 16),
                            1 << 30, None) == -3
    assert L.swin_wattn_index_map(ctypes.byref(d), None, None) == -1


def test_workspace_sizes_are_modest(L):
    for wl in WORKLOADS.values():
        n = sb.swin_wattn_workspace_size(sb.desc_for(wl))
        assert 256 <= n < 512 * 2**20, (wl.name, n)


def _a256(x):
    return (x + 255) // 256 * 256


@pytest.mark.parametrize("name", ["ragged-90x180-w8", "twelfth-degree-256x544-w8",
                                  "downsampled-128x272-w16", "small-patch-2x512x1088-w8",
                                  "tiny-16x16-w4"])
def test_workspace_size_follows_the_documented_layout(L, name):
    """Tensor-core families: 256-byte header, the transposed bias table
    [heads][bins padded to 4] fp32 and the exact bias-gradient sums
    [heads][bins padded][9 limbs + 1 flag] int64, each region 256-byte
    aligned. Portable
    kernels: header, per-row partials (3 floats per window slot and head) and
    per-window bias-gradient partials."""
    wl = WORKLOADS[name]
    d = sb.desc_for(wl)
    bins = (2 * wl.win - 1) ** 2
    bp = (bins + 3) // 4 * 4
    if sb.swin_wattn_path(d) in (1, 2, 3):
        want = 256 + _a256(wl.heads * bp * 4) + _a256(wl.heads * bp * 10 * 8)
    else:
        hp = -(-wl.H // wl.win) * wl.win
        wp = -(-wl.W // wl.win) * wl.win
        n_win = wl.B * (hp // wl.win) * (wp // wl.win)
        want = 256 + _a256(n_win * wl.heads * wl.win ** 2 * 3 * 4) + _a256(n_win * wl.heads * bp * 4)
    assert sb.swin_wattn_workspace_size(d) == want


def test_strerror_covers_every_status(L):
    for s in range(-5, 1):
        assert sb.swin_wattn_strerror(s) != "unknown status"


@pytest.mark.parametrize("win,hd,path", [((16, 16), 64, 3), ((32, 32), 128, 4)])
def test_row_band_entry_points_take_only_64_token_windows(L, win, hd, path):
    """A row band needs the 64-token kernels' halo boxes; other families are
    refused on the host, before any pointer is touched (these are fake,
    aligned host addresses)."""
    d = sb.make_desc(1, 64, 96, win, (win[0] // 2, win[1] // 2), 2, hd, "bf16")
    assert sb.swin_wattn_path(d) == path
    fake = ctypes.c_void_p(1 << 20)
    halo = sb.SwinWattnHalo(0, fake, fake, fake, fake, fake, None, fake, fake, fake)
    rc = L.swin_wattn_fwd_band(ctypes.byref(d), ctypes.byref(halo), fake, fake, fake, fake, fake,
                               None, fake, ctypes.c_size_t(1 << 30), None)
    assert rc == -2   # SWIN_ERR_UNSUPPORTED
    rc = L.swin_wattn_bwd_band(ctypes.byref(d), ctypes.byref(halo), fake, fake, fake, fake, fake,
                               fake, fake, fake, fake, fake, ctypes.c_size_t(1 << 30), None)
    assert rc == -2   # SWIN_ERR_UNSUPPORTED


def test_1024_token_workspace_adds_the_rows_statistics(L):
    """Path 4's workspace: the header, the bias table [heads][bins rounded up
    to 4] fp32, the exact bias-gradient sums (10 int64 words per head and
    bin), then L and D (float2) of every query of every window and head, each
    part rounded up to 256 bytes; the sums sit where swin_wattn_dbias_sums
    says."""
    a256 = lambda x: (x + 255) // 256 * 256
    for (H, W, heads, hd) in [(64, 96, 2, 128), (256, 544, 8, 128), (20, 24, 3, 64)]:
        d = sb.make_desc(1, H, W, (32, 32), (16, 16), heads, hd, "bf16")
        assert sb.swin_wattn_path(d) == 4
        bp = (63 * 63 + 3) // 4 * 4
        n_win = (-(-H // 32)) * (-(-W // 32))
        want = 256 + a256(heads * bp * 4) + a256(heads * bp * 80) + a256(n_win * heads * 1024 * 8)
        assert sb.swin_wattn_workspace_size(d) == want
        off, nbytes = ctypes.c_size_t(0), ctypes.c_size_t(0)
        assert L.swin_wattn_dbias_sums(ctypes.byref(d), ctypes.byref(off), ctypes.byref(nbytes)) == 0
        assert off.value == 256 + a256(heads * bp * 4) and nbytes.value == heads * bp * 80
