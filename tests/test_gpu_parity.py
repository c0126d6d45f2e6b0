"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs, element by element, plus bit-exact layout checks and
invariants. Acceptance bar: index and layout work bit-exact; fp32 max relative
error <= 1e-5 (normwise); bf16 max|gpu - ref| / RMS(ref) <= 2e-2 per tensor."""
import numpy as np
import pytest
import torch

import oracle
from shifted_window_attention_pad_b200 import WORKLOADS, binding as sb
from shifted_window_attention_pad_b200.synth import make_inputs, as_f64
from shifted_window_attention_pad_b200.workloads import Workload

from gpu_helpers import BF16_TOL, F32_TOL, compare, oracle_shape, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from shifted_window_attention_pad_b200 import build
    build.build()
    assert torch.cuda.is_available()


def tol(dtype):
    return F32_TOL if dtype == "f32" else BF16_TOL


# ---------------------------------------------------------------------------
# Layout stage: bit-exact
# ---------------------------------------------------------------------------
SWEEP = [(H, W, w, s) for (H, W) in [(1, 1), (5, 7), (16, 16), (17, 40), (40, 3), (90, 180)]
         for (w, s) in [(1, 0), (2, 1), (4, 2), (7, 3), (8, 4), (8, 0)]]


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_index_map_bit_exact_on_workload_shapes(name):
    wl = WORKLOADS[name]
    d = sb.desc_for(wl)
    gpu = sb.swin_wattn_index_map(d).cpu().numpy().reshape(wl.B, -1, wl.win * wl.win)
    ref = oracle.index_map(oracle_shape(d))
    assert np.array_equal(gpu.astype(np.int64), ref)


@pytest.mark.parametrize("H,W,w,s", SWEEP)
def test_index_map_bit_exact_sweep(H, W, w, s):
    d = sb.make_desc(2, H, W, w, s, 1, 8, "f32")
    gpu = sb.swin_wattn_index_map(d).cpu().numpy().reshape(2, -1, w * w)
    assert np.array_equal(gpu.astype(np.int64), oracle.index_map(oracle_shape(d)))


# The same bit-exact bar for the layout stage as the tcgen05 kernels run it:
# their TMA boxes (seam windows split into sub-boxes), the row order those
# boxes leave in shared memory and the per-row token and region each kernel
# derives. Every description here runs on those kernels (path 1).
FAST_LAYOUT = ([(1, H, W, (8, 8), (s, s), 3, hd) for (H, W) in [(1, 1), (5, 7), (16, 16), (17, 40),
                                                                (40, 3), (90, 180)]
                for s in (4, 0) for hd in (32, 64, 128)] +
               [(2, 18, 30, win, sh, 2, 64) for (win, sh) in [((4, 16), (2, 8)), ((16, 4), (8, 2)),
                                                                ((2, 32), (1, 16)), ((4, 16), (0, 0))]])


def _check_layout(d):
    assert sb.swin_wattn_path(d) == 1
    m, lab = sb.swin_wattn_layout_map(d)
    torch.cuda.synchronize()
    s = oracle_shape(d)
    ref = oracle.index_map(s)
    got = m.cpu().numpy().reshape(ref.shape).astype(np.int64)
    assert not np.any(got == -2)
    assert np.array_equal(got, ref)
    rl = oracle.region_labels(s)
    lab = lab.cpu().numpy().reshape(d.B, -1, d.win_h * d.win_w)
    for b in range(d.B):
        assert np.array_equal(lab[b], rl)


@pytest.mark.parametrize("case", FAST_LAYOUT, ids=lambda c: "%dx%dx%d-w%dx%d-s%dx%d-hd%d" % (
    c[0], c[1], c[2], *c[3], *c[4], c[6]))
def test_tcgen05_layout_stage_bit_exact(case):
    B, H, W, win, shift, heads, hd = case
    _check_layout(sb.make_desc(B, H, W, win, shift, heads, hd, "bf16"))


@pytest.mark.parametrize("name", ["ragged-90x180-w8", "twelfth-degree-256x544-w8",
                                  "small-patch-2x512x1088-w8"])
def test_tcgen05_layout_stage_bit_exact_on_workloads(name):
    _check_layout(sb.desc_for(WORKLOADS[name]))


@pytest.mark.parametrize("valid", [(256, 540), (251, 537)])
def test_tcgen05_layout_stage_with_a_valid_extent(valid):
    """The 1/12-degree token grid whose last columns (or rows) cover only
    padded field pixels: those slots read as padding."""
    wl = WORKLOADS["twelfth-degree-256x544-w8"]
    _check_layout(sb.make_desc(1, wl.H, wl.W, 8, 4, 2, 64, "bf16", valid=valid))


# ---------------------------------------------------------------------------
# Valid extent: stored tokens over padded field pixels (all kernel families)
# ---------------------------------------------------------------------------
VALID = [
    (1, Workload("valid-tcgen05", 2, 40, 56, 8, 4, 3, 64, "bf16", 71, valid=(37, 50))),
    (3, Workload("valid-tcgen05-w16", 1, 40, 52, 16, 8, 2, 64, "bf16", 72, valid=(35, 47))),
    (2, Workload("valid-warp-mma", 1, 40, 52, 16, 8, 2, 64, "bf16", 75, valid=(33, 49))),
    (0, Workload("valid-portable", 1, 13, 18, 4, 2, 2, 16, "f32", 73, valid=(11, 15))),
    (1, Workload("valid-1/12-degree-field", 1, 256, 544, 8, 4, 4, 64, "bf16", 74,
                 valid=sb.field_valid_extent(2041, 4320, 8))),
    (4, Workload("valid-tcgen05-w32", 1, 64, 96, 32, 16, 2, 128, "bf16", 76, valid=(61, 90))),
]


@pytest.mark.parametrize("case", VALID, ids=lambda c: c[1].name)
def test_valid_extent_parity(case):
    path, wl = case
    d = sb.desc_for(wl, flags=sb.SWIN_FLAG_FORCE_TILED if path == 2 else 0)
    assert sb.swin_wattn_path(d) == path
    inp = make_inputs(wl)
    gpu = run_gpu(d, inp)
    ref = run_oracle(d, inp)
    vh, vw = wl.valid
    for n in ("o", "lse", "dq", "dk", "dv"):
        g = gpu[n].cpu()
        assert torch.all(g[:, vh:] == 0) and torch.all(g[:, :, vw:] == 0), n
    errs = compare(gpu, ref, wl.dtype)
    print(wl.name, errs)
    for n, e in errs.items():
        assert e <= tol(wl.dtype), (wl.name, n, e)


# ---------------------------------------------------------------------------
# Parity on the five workloads
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["tiny-16x16-w4", "ragged-90x180-w8",
                                  "twelfth-degree-256x544-w8", "downsampled-128x272-w16"])
def test_parity_full(name):
    wl = WORKLOADS[name]
    inp = make_inputs(wl)
    d = sb.desc_for(wl)
    gpu = run_gpu(d, inp)
    ref = run_oracle(d, inp)
    errs = compare(gpu, ref, wl.dtype)
    print(name, "path", sb.swin_wattn_path(d), errs)
    assert set(errs) == {"o", "lse", "dq", "dk", "dv", "dT"}
    for n, e in errs.items():
        assert e <= tol(wl.dtype), (name, n, e)


def test_parity_small_patch_two_heads():
    """Batch 2 x 512 x 1088, 12 heads: the whole problem runs on the GPU; heads 0
    and 7 (heads are independent) are checked against the oracle in full."""
    wl = WORKLOADS["small-patch-2x512x1088-w8"]
    inp = make_inputs(wl)
    d = sb.desc_for(wl)
    gpu = run_gpu(d, inp, want_lse=False)
    for h in (0, 7):
        sub = {n: inp[n][:, :, :, h:h + 1].contiguous() for n in ("q", "k", "v", "dout")}
        sub["table"] = inp["table"][:, h:h + 1].contiguous()
        ds = sb.make_desc(wl.B, wl.H, wl.W, wl.win, wl.shift, 1, wl.head_dim, wl.dtype)
        ref = run_oracle(ds, sub)
        g = {n: gpu[n][:, :, :, h:h + 1] for n in ("o", "dq", "dk", "dv")}
        g["dT"] = gpu["dT"][:, h:h + 1]
        errs = compare(g, ref, wl.dtype)
        print("head", h, errs)
        for n, e in errs.items():
            assert e <= BF16_TOL, (h, n, e)


def test_generic_kernels_bf16_parity():
    wl = WORKLOADS["ragged-90x180-w8"]
    inp = make_inputs(wl)
    d = sb.desc_for(wl, flags=sb.SWIN_FLAG_FORCE_GENERIC)
    assert sb.swin_wattn_path(d) == 0
    errs = compare(run_gpu(d, inp), run_oracle(d, inp), "bf16")
    for n, e in errs.items():
        assert e <= BF16_TOL, (n, e)


# Shapes that exercise the fast path's edges: non-square windows, head_dim 32,
# a grid smaller than one window, no shift, an odd window count (half-empty
# tile), batch > 1.
EDGE = [
    Workload("edge-a", 2, 20, 28, 8, 4, 3, 64, "bf16", 11),
    Workload("edge-b", 1, 5, 6, 8, 4, 2, 64, "bf16", 12),
    Workload("edge-c", 1, 24, 40, 8, 0, 2, 32, "bf16", 13),
    Workload("edge-d", 3, 9, 17, 8, 4, 1, 32, "bf16", 14),
]


@pytest.mark.parametrize("wl", EDGE, ids=lambda w: w.name)
def test_fast_path_edges(wl):
    inp = make_inputs(wl)
    d = sb.desc_for(wl)
    assert sb.swin_wattn_path(d) == 1
    errs = compare(run_gpu(d, inp), run_oracle(d, inp), "bf16")
    print(wl.name, errs)
    for n, e in errs.items():
        assert e <= BF16_TOL, (wl.name, n, e)


@pytest.mark.parametrize("win,shift", [((4, 16), (2, 8)), ((16, 4), (8, 2)), ((2, 32), (1, 16))])
def test_fast_path_non_square_windows(win, shift):
    B, H, W, heads, hd = 1, 18, 30, 2, 64
    d = sb.make_desc(B, H, W, win, shift, heads, hd, "bf16")
    wl = Workload("ns", B, H, W, win[0], shift[0], heads, hd, "bf16", 21)
    inp = make_inputs(wl, shape_override=(B, H, W, heads, hd))
    nb = (2 * win[0] - 1) * (2 * win[1] - 1)
    inp["table"] = torch.from_numpy(
        np.random.Generator(np.random.PCG64(5)).standard_normal((nb, heads)).astype(np.float32) * 0.02)
    assert sb.swin_wattn_path(d) == 1
    errs = compare(run_gpu(d, inp), run_oracle(d, inp), "bf16")
    for n, e in errs.items():
        assert e <= BF16_TOL, (win, n, e)


# ---------------------------------------------------------------------------
# Warp-level tensor-core kernels (path 2): windows of up to 256 tokens
# ---------------------------------------------------------------------------
# (B, H, W, window, shift, heads, head_dim, seed): 16 x 16 windows on a padded
# grid, window sizes that fill 64, 128 and 256 slots only partly, head_dim 32,
# batch > 1, no shift; every (slots, head_dim) kernel instance meets both plain
# windows (no pad, one shift region) and masked ones.
TILED = [
    (1, 40, 52, (16, 16), (8, 8), 2, 64, 31),
    (2, 23, 30, (7, 7), (3, 3), 2, 64, 32),
    (1, 30, 41, (8, 12), (4, 6), 3, 32, 33),
    (1, 37, 26, (12, 12), (6, 6), 2, 32, 34),
    (1, 32, 48, (16, 8), (0, 0), 2, 64, 35),
    (1, 20, 36, (4, 16), (2, 5), 2, 64, 36),
    (1, 32, 48, (16, 16), (8, 8), 3, 32, 37),
]


@pytest.mark.parametrize("case", TILED, ids=lambda c: "%dx%d-w%dx%d-hd%d" % (c[1], c[2], *c[3], c[6]))
def test_tiled_path_parity(case):
    B, H, W, win, shift, heads, hd, seed = case
    # (256-token windows go to the tcgen05 kernels unless the warp-MMA ones are forced)
    d = sb.make_desc(B, H, W, win, shift, heads, hd, "bf16", flags=sb.SWIN_FLAG_FORCE_TILED)
    assert sb.swin_wattn_path(d) == 2
    wl = Workload("tiled", B, H, W, win[0], shift[0], heads, hd, "bf16", seed)
    inp = make_inputs(wl, shape_override=(B, H, W, heads, hd))
    nb = (2 * win[0] - 1) * (2 * win[1] - 1)
    inp["table"] = torch.from_numpy(np.random.Generator(np.random.PCG64(seed)).standard_normal(
        (nb, heads)).astype(np.float32) * 0.02)
    errs = compare(run_gpu(d, inp), run_oracle(d, inp), "bf16")
    print(case, errs)
    for n, e in errs.items():
        assert e <= BF16_TOL, (case, n, e)


# ---------------------------------------------------------------------------
# tcgen05 kernels for 256-token windows (path 3)
# ---------------------------------------------------------------------------
# (B, H, W, window, shift, heads, head_dim, seed): a padded grid with both
# seams, no shift, head_dim 32, batch > 1, a grid smaller than one window,
# 8 x 32 windows (seam sub-boxes of 8 x 16 tokens), the 16 x 16 window row of
# the downsampled grid
WIDE = [
    (1, 40, 52, (16, 16), (8, 8), 2, 64, 81),
    (1, 32, 48, (16, 16), (0, 0), 2, 64, 82),
    (2, 36, 30, (16, 16), (8, 8), 3, 32, 83),
    (1, 11, 13, (16, 16), (8, 8), 2, 64, 84),
    (1, 24, 70, (8, 32), (4, 16), 2, 64, 85),
    (1, 16, 272, (16, 16), (8, 8), 4, 64, 86),
]


@pytest.mark.parametrize("case", WIDE, ids=lambda c: "%dx%dx%d-w%dx%d-s%d-hd%d" % (
    c[0], c[1], c[2], *c[3], c[4][0], c[6]))
def test_wide_path_parity(case):
    B, H, W, win, shift, heads, hd, seed = case
    d = sb.make_desc(B, H, W, win, shift, heads, hd, "bf16")
    assert sb.swin_wattn_path(d) == 3
    wl = Workload("wide", B, H, W, win[0], shift[0], heads, hd, "bf16", seed)
    inp = make_inputs(wl, shape_override=(B, H, W, heads, hd))
    nb = (2 * win[0] - 1) * (2 * win[1] - 1)
    inp["table"] = torch.from_numpy(np.random.Generator(np.random.PCG64(seed)).standard_normal(
        (nb, heads)).astype(np.float32) * 0.02)
    errs = compare(run_gpu(d, inp), run_oracle(d, inp), "bf16")
    print(case, errs)
    for n, e in errs.items():
        assert e <= BF16_TOL, (case, n, e)


# ---------------------------------------------------------------------------
# tcgen05 kernels for 1024-token windows (path 4)
# ---------------------------------------------------------------------------
# (B, H, W, window, shift, heads, head_dim, seed): both seams at head_dim 128
# and 64, a padded grid, no shift, batch 2, a row shift whose seam splits a
# 128-token block (window row 18 of 32), the largest model's window at the
# 1/12-degree grid's width, a grid smaller than one window
LARGE = [
    (1, 64, 96, (32, 32), (16, 16), 2, 128, 91),
    (1, 40, 72, (32, 32), (16, 16), 1, 64, 92),
    (1, 32, 64, (32, 32), (0, 0), 2, 128, 93),
    (2, 64, 64, (32, 32), (16, 16), 1, 128, 94),
    (1, 64, 96, (32, 32), (14, 16), 1, 64, 95),
    (1, 32, 544, (32, 32), (16, 16), 1, 128, 96),
    (1, 20, 24, (32, 32), (16, 16), 2, 64, 97),
]


@pytest.mark.parametrize("case", LARGE, ids=lambda c: "%dx%dx%d-w%dx%d-s%dx%d-hd%d" % (
    c[0], c[1], c[2], *c[3], *c[4], c[6]))
def test_large_path_parity(case):
    B, H, W, win, shift, heads, hd, seed = case
    d = sb.make_desc(B, H, W, win, shift, heads, hd, "bf16")
    assert sb.swin_wattn_path(d) == 4
    wl = Workload("large", B, H, W, win[0], shift[0], heads, hd, "bf16", seed)
    inp = make_inputs(wl, shape_override=(B, H, W, heads, hd))
    nb = (2 * win[0] - 1) * (2 * win[1] - 1)
    inp["table"] = torch.from_numpy(np.random.Generator(np.random.PCG64(seed)).standard_normal(
        (nb, heads)).astype(np.float32) * 0.02)
    errs = compare(run_gpu(d, inp), run_oracle(d, inp), "bf16")
    print(case, errs)
    for n, e in errs.items():
        assert e <= BF16_TOL, (case, n, e)


def test_large_windows_on_the_table5_grid_two_heads():
    """Table V's largest window on the 1/12-degree token grid: 256 x 544
    tokens, 32 x 32 windows, shift 16, 8 heads x 128, the bench workload's
    launch. The whole problem runs on the GPU; heads 0 and 7 are checked
    against the oracle in full, and the backward repeats bitwise."""
    wl = WORKLOADS["table5-large-256x544-8x128-w32"]
    inp = make_inputs(wl)
    d = sb.desc_for(wl)
    assert sb.swin_wattn_path(d) == 4
    gpu = run_gpu(d, inp, want_lse=False)
    again = run_gpu(d, inp, want_lse=False)
    for n in ("o", "dq", "dk", "dv", "dT"):
        assert torch.equal(gpu[n], again[n]), n
    for h in (0, 7):
        sub = {n: inp[n][:, :, :, h:h + 1].contiguous() for n in ("q", "k", "v", "dout")}
        sub["table"] = inp["table"][:, h:h + 1].contiguous()
        ds = sb.make_desc(wl.B, wl.H, wl.W, wl.win, wl.shift, 1, wl.head_dim, wl.dtype)
        g = {n: gpu[n][:, :, :, h:h + 1] for n in ("o", "dq", "dk", "dv")}
        g["dT"] = gpu["dT"][:, h:h + 1]
        for n, e in compare(g, run_oracle(ds, sub), "bf16").items():
            assert e <= BF16_TOL, (h, n, e)


@pytest.mark.parametrize("name", ["ragged-90x180-w8", "small-patch-2x512x1088-w8"])
def test_tiled_path_forced_on_window64_workloads(name):
    """The warp-MMA kernels on the 8 x 8-window workloads the tcgen05 kernels
    normally take (ragged grid in full; the large batch-2 grid on two heads)."""
    wl = WORKLOADS[name]
    inp = make_inputs(wl)
    d = sb.desc_for(wl, flags=sb.SWIN_FLAG_FORCE_TILED)
    assert sb.swin_wattn_path(d) == 2
    gpu = run_gpu(d, inp, want_lse=(wl.B == 1))
    if wl.B == 1:
        errs = compare(gpu, run_oracle(d, inp), "bf16")
        for n, e in errs.items():
            assert e <= BF16_TOL, (n, e)
        return
    for h in (0, 11):
        sub = {n: inp[n][:, :, :, h:h + 1].contiguous() for n in ("q", "k", "v", "dout")}
        sub["table"] = inp["table"][:, h:h + 1].contiguous()
        ds = sb.make_desc(wl.B, wl.H, wl.W, wl.win, wl.shift, 1, wl.head_dim, wl.dtype)
        g = {n: gpu[n][:, :, :, h:h + 1] for n in ("o", "dq", "dk", "dv")}
        g["dT"] = gpu["dT"][:, h:h + 1]
        for n, e in compare(g, run_oracle(ds, sub), "bf16").items():
            assert e <= BF16_TOL, (h, n, e)


@pytest.mark.parametrize("path", [3, 2])
def test_backward_of_256_token_windows_is_deterministic(path):
    wl = WORKLOADS["downsampled-128x272-w16"]
    inp = make_inputs(wl)
    d = sb.desc_for(wl, flags=sb.SWIN_FLAG_FORCE_TILED if path == 2 else 0)
    assert sb.swin_wattn_path(d) == path
    a = run_gpu(d, inp, want_lse=False)
    b = run_gpu(d, inp, want_lse=False)
    for n in ("o", "dq", "dk", "dv", "dT"):
        assert torch.equal(a[n], b[n]), n


# ---------------------------------------------------------------------------
# Exact cases and invariants
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_hand_example_isolated_tokens_exact_on_gpu(dtype):
    """4x4 grid, 2x2 windows, shift 1: the corner window's four tokens each sit
    in their own region, so o = v, dq = dk = 0 and dv = dO exactly."""
    wl = Workload("hand", 1, 4, 4, 2, 1, 3, 8, dtype, 3)
    inp = make_inputs(wl)
    d = sb.desc_for(wl)
    gpu = run_gpu(d, inp)
    for tok in (15, 12, 3, 0):
        y, x = divmod(tok, 4)
        assert torch.equal(gpu["o"][0, y, x].cpu(), inp["v"][0, y, x])
        assert torch.all(gpu["dq"][0, y, x] == 0) and torch.all(gpu["dk"][0, y, x] == 0)
        assert torch.equal(gpu["dv"][0, y, x].cpu(), inp["dout"][0, y, x])


def test_other_region_keys_do_not_reach_a_query_bit_exact():
    """Corner window of an unpadded 32 x 48 grid (four 4 x 4 shift regions):
    change k and v of one token of one region; queries of the other regions in
    that window keep identical bits, those of its own region change."""
    wl = Workload("iso", 1, 32, 48, 8, 4, 2, 64, "bf16", 7)
    inp = make_inputs(wl)
    d = sb.desc_for(wl)
    s = oracle_shape(d)
    m = oracle.index_map(s)[0]
    lab = oracle.region_labels(s)
    win = m.shape[0] - 1                       # bottom-right corner window
    src, labels = m[win], lab[win]
    tgt = next(i for i in range(len(src)) if src[i] >= 0)
    others = [src[i] for i in range(len(src)) if src[i] >= 0 and labels[i] != labels[tgt]]
    same = [src[i] for i in range(len(src)) if src[i] >= 0 and labels[i] == labels[tgt]
            and i != tgt]
    assert others and same
    o1 = run_gpu(d, inp, backward=False)["o"].reshape(-1, wl.heads, wl.head_dim).cpu()
    inp2 = dict(inp)
    for n in ("k", "v"):
        t = inp[n].clone().reshape(-1, wl.heads, wl.head_dim)
        t[src[tgt]] += 3.0
        inp2[n] = t.reshape(inp[n].shape)
    o2 = run_gpu(d, inp2, backward=False)["o"].reshape(-1, wl.heads, wl.head_dim).cpu()
    assert torch.equal(o1[others], o2[others])
    assert not torch.equal(o1[same], o2[same])


def test_bias_gradient_sums_to_zero_and_backward_is_deterministic():
    wl = WORKLOADS["twelfth-degree-256x544-w8"]
    inp = make_inputs(wl)
    d = sb.desc_for(wl)
    a = run_gpu(d, inp, want_lse=False)
    b = run_gpu(d, inp, want_lse=False)
    for n in ("o", "dq", "dk", "dv", "dT"):
        assert torch.equal(a[n], b[n]), n
    dT = as_f64(a["dT"])
    assert np.all(np.abs(dT.sum(axis=0)) <= 1e-3 * np.abs(dT).sum(axis=0) + 1e-6)


@pytest.mark.parametrize("path", [1, 4])
def test_bounded_wait_reports_timeout_and_context_survives(path):
    """A wait on a barrier that nothing arrives on runs out after ~1 ms: the call
    reports SWIN_ERR_TIMEOUT through the workspace status word, and the next
    call on the same context works (64-token and 1024-token kernels)."""
    wl = (WORKLOADS["ragged-90x180-w8"] if path == 1 else
          Workload("w32", 1, 40, 72, 32, 16, 2, 64, "bf16", 43))
    inp = make_inputs(wl)
    assert sb.swin_wattn_path(sb.desc_for(wl)) == path
    dev = "cuda"
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "dout"))
    T = inp["table"].to(dev)
    d = sb.desc_for(wl, flags=sb.SWIN_FLAG_TEST_TIMEOUT)
    ws = sb.new_workspace(d)
    out = torch.empty_like(q)
    sb.swin_wattn_fwd(d, q, k, v, T, out, None, ws)
    assert sb.swin_wattn_poll_status(ws) == sb.SWIN_ERR_TIMEOUT
    dq, dk, dv, dT = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(T)
    sb.swin_wattn_bwd(d, q, k, v, T, do, dq, dk, dv, dT, ws)
    assert sb.swin_wattn_poll_status(ws) == sb.SWIN_ERR_TIMEOUT
    assert sb.swin_wattn_poll_status(ws) == 0
    d_ok = sb.desc_for(wl)
    gpu = run_gpu(d_ok, inp)
    ref = run_oracle(d_ok, inp)
    for n, e in compare(gpu, ref, "bf16").items():
        assert e <= BF16_TOL, (n, e)


# ---------------------------------------------------------------------------
# head_dim 128 on the tcgen05 kernels (TERRA page, Table V: every model size
# uses 128-channel heads): two channel halves per TMA box, P kept in TMEM as
# the A operand of P V, a one-stage, one-slot backward
# ---------------------------------------------------------------------------
HD128 = [
    Workload("hd128-ragged-90x180", 1, 90, 180, 8, 4, 2, 128, "bf16", 81),
    Workload("hd128-batch2-20x28", 2, 20, 28, 8, 4, 3, 128, "bf16", 82),
    Workload("hd128-noshift-24x40", 1, 24, 40, 8, 0, 2, 128, "bf16", 83),
    Workload("hd128-tiny-5x6", 1, 5, 6, 8, 4, 1, 128, "bf16", 84),
]


@pytest.mark.parametrize("wl", HD128, ids=lambda w: w.name)
def test_head_dim_128_parity(wl):
    inp = make_inputs(wl)
    d = sb.desc_for(wl)
    assert sb.swin_wattn_path(d) == 1
    errs = compare(run_gpu(d, inp), run_oracle(d, inp), "bf16")
    print(wl.name, errs)
    assert set(errs) == {"o", "lse", "dq", "dk", "dv", "dT"}
    for n, e in errs.items():
        assert e <= BF16_TOL, (wl.name, n, e)


@pytest.mark.parametrize("win,shift", [((4, 16), (2, 8)), ((16, 4), (8, 2))])
def test_head_dim_128_non_square_windows(win, shift):
    B, H, W, heads, hd = 1, 18, 30, 2, 128
    d = sb.make_desc(B, H, W, win, shift, heads, hd, "bf16")
    assert sb.swin_wattn_path(d) == 1
    wl = Workload("ns128", B, H, W, win[0], shift[0], heads, hd, "bf16", 85)
    inp = make_inputs(wl, shape_override=(B, H, W, heads, hd))
    nb = (2 * win[0] - 1) * (2 * win[1] - 1)
    inp["table"] = torch.from_numpy(
        np.random.Generator(np.random.PCG64(6)).standard_normal((nb, heads)).astype(np.float32) * 0.02)
    errs = compare(run_gpu(d, inp), run_oracle(d, inp), "bf16")
    for n, e in errs.items():
        assert e <= BF16_TOL, (win, n, e)


def test_head_dim_128_table5_grid_two_heads():
    """The 1/12-degree token grid with Table V's head size: 256 x 544 tokens,
    8 heads x 128 (d = 1024). The whole problem runs on the GPU; heads 0 and 5
    are checked against the oracle in full, and the backward repeats bitwise."""
    wl = Workload("table5-256x544-8x128", 1, 256, 544, 8, 4, 8, 128, "bf16", 86)
    inp = make_inputs(wl)
    d = sb.desc_for(wl)
    assert sb.swin_wattn_path(d) == 1
    gpu = run_gpu(d, inp, want_lse=False)
    again = run_gpu(d, inp, want_lse=False)
    for n in ("o", "dq", "dk", "dv", "dT"):
        assert torch.equal(gpu[n], again[n]), n
    for h in (0, 5):
        sub = {n: inp[n][:, :, :, h:h + 1].contiguous() for n in ("q", "k", "v", "dout")}
        sub["table"] = inp["table"][:, h:h + 1].contiguous()
        ds = sb.make_desc(wl.B, wl.H, wl.W, wl.win, wl.shift, 1, wl.head_dim, wl.dtype)
        g = {n: gpu[n][:, :, :, h:h + 1] for n in ("o", "dq", "dk", "dv")}
        g["dT"] = gpu["dT"][:, h:h + 1]
        for n, e in compare(g, run_oracle(ds, sub), "bf16").items():
            assert e <= BF16_TOL, (h, n, e)
