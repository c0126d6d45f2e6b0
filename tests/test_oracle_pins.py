"""Pins of the fp64 CPU oracle against facts that do not come from the oracle itself.

Each test names what fixes the expected value: a hand enumeration (tests/golden),
an identity, a closed form, a library routine (torch scaled-dot-product attention
and autograd in fp64) for the special cases that reduce to plain attention, a
brute-force per-token formulation on tiny grids, or central finite differences.
Page cited: "TERRA: A Hierarchical Parallel Training and Memory Orchestration
Framework for High-Resolution AI-based Earth Modeling", Abstract (window-based
Swin attention with shifted-window execution) and Table I (padded resolution).
"""
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, scale=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * scale


def problem(B, H, W, win, shift, heads, hd, seed=0, tscale=0.3):
    s = oracle.make_shape(B, H, W, win, shift, heads, hd)
    g = (B, H, W, heads, hd)
    q, k, v, do = (rnd(g, seed + i) for i in range(4))
    T = rnd((oracle.n_bins(s), heads), seed + 9, tscale)
    return s, q, k, v, T, do


SHAPES = [  # (H, W, (win_h, win_w), (shift_h, shift_w))
    (4, 4, 2, 1), (8, 8, 4, 2), (6, 7, 4, 2), (9, 5, 3, 1), (5, 13, (2, 4), (1, 3)),
    (16, 16, 4, 0), (7, 7, 8, 4), (1, 1, 1, 0), (3, 10, (3, 5), (2, 0)),
]


# ---------------------------------------------------------------------------
# Layout: identities and the hand-enumerated example (bit-exact)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("H,W,win,shift", SHAPES)
def test_partition_then_reverse_is_identity(H, W, win, shift):
    s = oracle.make_shape(1, H, W, win, shift, 1, 1)
    Hp, Wp = oracle.padded_hw(s)
    grid = np.random.Generator(np.random.PCG64(H * 31 + W)).integers(-2**40, 2**40, (Hp, Wp))
    assert np.array_equal(oracle.roundtrip(s, grid, "partition"), grid)


@pytest.mark.parametrize("H,W,win,shift", SHAPES)
def test_roll_then_unroll_is_identity(H, W, win, shift):
    s = oracle.make_shape(1, H, W, win, shift, 1, 1)
    Hp, Wp = oracle.padded_hw(s)
    grid = np.random.Generator(np.random.PCG64(H * 17 + W)).integers(-2**40, 2**40, (Hp, Wp))
    assert np.array_equal(oracle.roundtrip(s, grid, "roll"), grid)


@pytest.mark.parametrize("H,W,win,shift", SHAPES)
def test_index_map_is_a_bijection_onto_valid_tokens(H, W, win, shift):
    B = 2
    s = oracle.make_shape(B, H, W, win, shift, 1, 1)
    Hp, Wp = oracle.padded_hw(s)
    m = oracle.index_map(s)
    ids = m[m >= 0]
    assert np.array_equal(np.sort(ids), np.arange(B * H * W))
    assert int((m < 0).sum()) == B * (Hp * Wp - H * W)


def _brute_rolled_source(H, W, Hp, Wp, wh, ww, sh, sw, b):
    """Per-token formulation: token (y, x) sits at rolled ((y-s_h) mod H^, (x-s_w) mod W^)."""
    nWx = Wp // ww
    m = -np.ones(((Hp // wh) * nWx, wh * ww), np.int64)
    for y in range(H):
        for x in range(W):
            yr, xr = (y - sh) % Hp, (x - sw) % Wp
            m[(yr // wh) * nWx + xr // ww, (yr % wh) * ww + xr % ww] = (b * H + y) * W + x
    return m


@pytest.mark.parametrize("H,W,win,shift", SHAPES)
def test_index_map_matches_per_token_formulation(H, W, win, shift):
    s = oracle.make_shape(2, H, W, win, shift, 1, 1)
    Hp, Wp = oracle.padded_hw(s)
    m = oracle.index_map(s)
    for b in range(2):
        exp = _brute_rolled_source(H, W, Hp, Wp, s.win_h, s.win_w, s.shift_h, s.shift_w, b)
        assert np.array_equal(m[b], exp)


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            left, right = line.split("|")
            vals = [int(t) for t in left.split()]
            rows.append((vals[0], vals[1:], [int(t) for t in right.split()]))
    return rows


def test_hand_example_index_map_and_regions():
    s = oracle.make_shape(1, 4, 4, 2, 1, 1, 1)
    m = oracle.index_map(s)[0]
    lab = oracle.region_labels(s)
    for win, ids, labels in _read_golden("hand_4x4_w2_s1.txt"):
        assert list(m[win]) == ids
        assert list(lab[win]) == labels


def test_hand_example_isolated_tokens_exact():
    """Window (1,1) of the hand example: four distinct regions, so every token is
    alone: o = v, dq = dk = 0, dv = dO exactly."""
    s, q, k, v, T, do = problem(1, 4, 4, 2, 1, 3, 5, seed=3)
    o, lse = oracle.forward(s, q, k, v, T)
    dq, dk, dv, dT = oracle.backward(s, q, k, v, T, do)
    for tok in (15, 12, 3, 0):
        y, x = divmod(tok, 4)
        assert np.array_equal(o[0, y, x], v[0, y, x])
        assert np.all(dq[0, y, x] == 0) and np.all(dk[0, y, x] == 0)
        assert np.array_equal(dv[0, y, x], do[0, y, x])


def test_hand_example_region_isolation_bit_exact():
    """Window (0,1) splits into {7, 11} and {4, 8}: changing k, v of token 4 must
    leave the outputs of tokens 7 and 11 bit-identical and change token 8's."""
    s, q, k, v, T, do = problem(1, 4, 4, 2, 1, 2, 4, seed=5)
    o1, _ = oracle.forward(s, q, k, v, T)
    k2, v2 = k.copy(), v.copy()
    k2[0, 1, 0] += 1.5
    v2[0, 1, 0] -= 2.0
    o2, _ = oracle.forward(s, q, k2, v2, T)
    assert np.array_equal(o1[0, 1, 3], o2[0, 1, 3]) and np.array_equal(o1[0, 2, 3], o2[0, 2, 3])
    assert not np.array_equal(o1[0, 2, 0], o2[0, 2, 0])


# ---------------------------------------------------------------------------
# Special cases that reduce to plain attention (torch fp64 library routines)
# ---------------------------------------------------------------------------
def _sdpa_heads(qt, kt, vt, mask=None):
    # qt: [heads, N, hd]
    return F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)


@pytest.mark.parametrize("H,W", [(6, 5), (4, 8), (3, 3), (32, 32)])
def test_one_window_no_shift_zero_bias_equals_sdpa(H, W):
    heads, hd = 2, 8
    s, q, k, v, T, do = problem(1, H, W, (H, W), 0, heads, hd, seed=11)
    T[:] = 0.0
    o, _ = oracle.forward(s, q, k, v, T)
    tq, tk, tv = (torch.from_numpy(a[0].reshape(H * W, heads, hd)).permute(1, 0, 2)
                  for a in (q, k, v))
    ref = _sdpa_heads(tq, tk, tv).permute(1, 0, 2).reshape(H, W, heads, hd).numpy()
    np.testing.assert_allclose(o[0], ref, rtol=0, atol=1e-12)


def test_one_window_with_padding_equals_sdpa_over_valid_tokens():
    """5x7 grid in one 8x8 window, no shift: pad keys get zero weight, so the
    result is plain attention over the 35 real tokens."""
    H, W, heads, hd = 5, 7, 3, 6
    s, q, k, v, T, do = problem(1, H, W, 8, 0, heads, hd, seed=12)
    T[:] = 0.0
    o, _ = oracle.forward(s, q, k, v, T)
    tq, tk, tv = (torch.from_numpy(a[0].reshape(H * W, heads, hd)).permute(1, 0, 2)
                  for a in (q, k, v))
    ref = _sdpa_heads(tq, tk, tv).permute(1, 0, 2).reshape(H, W, heads, hd).numpy()
    np.testing.assert_allclose(o[0], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("H,W,win", [(6, 5, (6, 5)), (5, 7, 8), (32, 32, 32), (20, 27, 32)])
def test_one_window_backward_equals_autograd(H, W, win):
    heads, hd = 2, 5
    s, q, k, v, T, do = problem(1, H, W, win, 0, heads, hd, seed=13)
    T[:] = 0.0
    dq, dk, dv, dT = oracle.backward(s, q, k, v, T, do)
    tq, tk, tv = (torch.from_numpy(a[0].reshape(H * W, heads, hd)).permute(1, 0, 2)
                  .clone().requires_grad_(True) for a in (q, k, v))
    out = _sdpa_heads(tq, tk, tv)
    g = torch.from_numpy(do[0].reshape(H * W, heads, hd)).permute(1, 0, 2)
    out.backward(g)
    for mine, t in ((dq, tq), (dk, tk), (dv, tv)):
        ref = t.grad.permute(1, 0, 2).reshape(H, W, heads, hd).numpy()
        np.testing.assert_allclose(mine[0], ref, rtol=0, atol=1e-11)


@pytest.mark.parametrize("dy,dx", [(1, -2), (-3, 1), (0, 2)])
def test_relative_bias_direction_closed_form(dy, dx):
    """q = 0 leaves only the bias in the logits. With one table entry, for the
    offset (query slot - key slot) = (dy, dx), set to 60 and the rest 0, each
    query whose key at that offset exists sends all but e^-60 of its weight there:
    o(i) = v(i - (dy, dx)). A table read with the offset reversed or its axes
    swapped fails this."""
    wh, ww, heads, hd = 4, 5, 1, 3
    s, q, k, v, T, do = problem(1, wh, ww, (wh, ww), 0, heads, hd, seed=14)
    q[:] = 0.0
    T[:] = 0.0
    T[(dy + wh - 1) * (2 * ww - 1) + (dx + ww - 1), 0] = 60.0
    o, _ = oracle.forward(s, q, k, v, T)
    for iy in range(wh):
        for ix in range(ww):
            jy, jx = iy - dy, ix - dx
            if 0 <= jy < wh and 0 <= jx < ww:
                np.testing.assert_allclose(o[0, iy, ix, 0], v[0, jy, jx, 0], rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# Closed forms and invariants with shift and padding
# ---------------------------------------------------------------------------
def _swin_slice_labels(Hp, Wp, wh, ww, sh, sw):
    """Region image built the way the Swin scheme describes it: three slices per
    axis on the rolled grid, each (row slice, column slice) block one label."""
    img = np.zeros((Hp, Wp), np.int64)
    hs = [slice(0, Hp - wh), slice(Hp - wh, Hp - sh), slice(Hp - sh, Hp)] if sh else [slice(0, Hp)]
    ws = [slice(0, Wp - ww), slice(Wp - ww, Wp - sw), slice(Wp - sw, Wp)] if sw else [slice(0, Wp)]
    c = 0
    for a in hs:
        for b in ws:
            img[a, b] = c
            c += 1
    return img


@pytest.mark.parametrize("H,W,win,shift", [(6, 7, 4, 2), (9, 5, 3, 1), (4, 4, 2, 1),
                                           (5, 13, (2, 4), (1, 3)), (10, 12, 4, 2)])
def test_zero_logits_give_region_means(H, W, win, shift):
    """q = 0 and T = 0: every allowed key has the same logit, so o(i) is the mean of
    v over the keys that share query i's window and region and are not padding,
    and lse(i) = log(count)."""
    B, heads, hd = 2, 2, 3
    s, q, k, v, T, do = problem(B, H, W, win, shift, heads, hd, seed=21)
    q[:] = 0.0
    T[:] = 0.0
    o, lse = oracle.forward(s, q, k, v, T)
    Hp, Wp = oracle.padded_hw(s)
    img = _swin_slice_labels(Hp, Wp, s.win_h, s.win_w, s.shift_h, s.shift_w)
    nWx = Wp // s.win_w
    m = oracle.index_map(s)
    vflat = v.reshape(B * H * W, heads, hd)
    oflat = o.reshape(B * H * W, heads, hd)
    lflat = lse.reshape(B * H * W, heads)
    for b in range(B):
        for win_id in range(m.shape[1]):
            wy, wx = divmod(win_id, nWx)
            lab = np.array([img[wy * s.win_h + i // s.win_w, wx * s.win_w + i % s.win_w]
                            for i in range(s.win_h * s.win_w)])
            src = m[b, win_id]
            for i in range(len(src)):
                if src[i] < 0:
                    continue
                keys = [src[j] for j in range(len(src)) if src[j] >= 0 and lab[j] == lab[i]]
                np.testing.assert_allclose(oflat[src[i]], vflat[keys].mean(axis=0), atol=1e-13)
                np.testing.assert_allclose(lflat[src[i]], np.log(len(keys)), atol=1e-13)


def test_bias_constant_shift_leaves_output_unchanged():
    s, q, k, v, T, do = problem(1, 10, 12, 4, 2, 2, 4, seed=31)
    o1, _ = oracle.forward(s, q, k, v, T)
    o2, _ = oracle.forward(s, q, k, v, T + 3.25)
    np.testing.assert_allclose(o1, o2, atol=1e-12)


def test_bias_gradient_sums_to_zero_per_head():
    """Each softmax row's dS sums to zero, so every head's dT sums to zero."""
    s, q, k, v, T, do = problem(2, 10, 11, 4, 2, 3, 4, seed=32)
    dq, dk, dv, dT = oracle.backward(s, q, k, v, T, do)
    assert np.all(np.abs(dT.sum(axis=0)) <= 1e-11 * (1 + np.abs(dT).sum(axis=0)))
    assert np.abs(dT).max() > 1e-3


def test_batch_images_are_independent():
    """Each batch image is its own grid: image 0 of a batch of two gives the same
    bits as the same image alone."""
    s1, q, k, v, T, do = problem(1, 7, 6, 4, 2, 2, 3, seed=33)
    s2 = oracle.make_shape(2, 7, 6, 4, 2, 2, 3)
    q2 = np.concatenate([q, q[:, ::-1] * 0.5])
    k2 = np.concatenate([k, -k])
    v2 = np.concatenate([v, v])
    o1, _ = oracle.forward(s1, q, k, v, T)
    o2, _ = oracle.forward(s2, q2, k2, v2, T)
    assert np.array_equal(o1[0], o2[0])


@pytest.mark.parametrize("H,W,win,shift", [(6, 7, 4, 2), (5, 13, (2, 4), (1, 3)), (8, 8, 4, 2),
                                           (20, 18, 16, 8), (9, 14, (7, 7), (3, 3))])
def test_forward_matches_per_token_brute_force(H, W, win, shift):
    """Brute force straight from the per-token description: for a real token,
    the keys are the real tokens whose rolled position falls in the same window
    and the same region; logits scale*q.k + T[offset]."""
    B, heads, hd = 1, 2, 3
    s, q, k, v, T, do = problem(B, H, W, win, shift, heads, hd, seed=41)
    o, lse = oracle.forward(s, q, k, v, T)
    Hp, Wp = oracle.padded_hw(s)
    wh, ww, sh, sw = s.win_h, s.win_w, s.shift_h, s.shift_w
    img = _swin_slice_labels(Hp, Wp, wh, ww, sh, sw)
    scale = hd ** -0.5
    toks = [(y, x) for y in range(H) for x in range(W)]
    roll = {t: ((t[0] - sh) % Hp, (t[1] - sw) % Wp) for t in toks}
    for h in range(heads):
        for t in toks:
            yr, xr = roll[t]
            keys = [u for u in toks if roll[u][0] // wh == yr // wh and roll[u][1] // ww == xr // ww
                    and img[roll[u]] == img[yr, xr]]
            logits = []
            for u in keys:
                dy = yr % wh - roll[u][0] % wh
                dx = xr % ww - roll[u][1] % ww
                logits.append(scale * np.dot(q[0, t[0], t[1], h], k[0, u[0], u[1], h]) +
                              T[(dy + wh - 1) * (2 * ww - 1) + dx + ww - 1, h])
            logits = np.array(logits)
            p = np.exp(logits - logits.max())
            p /= p.sum()
            ref = sum(pj * v[0, u[0], u[1], h] for pj, u in zip(p, keys))
            np.testing.assert_allclose(o[0, t[0], t[1], h], ref, atol=1e-13)


# ---------------------------------------------------------------------------
# Backward: central finite differences of the oracle forward
# ---------------------------------------------------------------------------
def _loss(s, q, k, v, T, G):
    o, _ = oracle.forward(s, q, k, v, T, want_lse=False)
    return float((o * G).sum())


@pytest.mark.parametrize("H,W,win,shift", [(6, 7, 4, 2), (4, 4, 2, 1), (5, 6, (2, 3), (1, 1)),
                                           (20, 18, 16, 8)])
def test_backward_matches_finite_differences(H, W, win, shift):
    B, heads, hd = 1, 2, 3
    s, q, k, v, T, G = problem(B, H, W, win, shift, heads, hd, seed=51)
    dq, dk, dv, dT = oracle.backward(s, q, k, v, T, G)
    eps = 1e-6
    rng = np.random.Generator(np.random.PCG64(7))
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv), ("T", T, dT)):
        flat = arr.reshape(-1)
        idxs = rng.choice(flat.size, size=min(flat.size, 24), replace=False)
        for i in idxs:
            old = flat[i]
            flat[i] = old + eps
            lp = _loss(s, q, k, v, T, G)
            flat[i] = old - eps
            lm = _loss(s, q, k, v, T, G)
            flat[i] = old
            fd = (lp - lm) / (2 * eps)
            an = grad.reshape(-1)[i]
            assert abs(fd - an) <= 2e-8 + 2e-7 * abs(an), (name, i, fd, an)


# ---------------------------------------------------------------------------
# The bf16 error measure of the parity tests
# ---------------------------------------------------------------------------
def test_bf16_measure_charges_computation_not_storage_rounding():
    """Rounding the exact result to bf16 costs (next to) nothing under the parity
    measure (but up to 0.04 RMS under the raw max|d|/RMS), while a real
    computational error of 3% of the RMS on one element is caught. (torch rounds
    fp64 -> bf16 through fp32, a double rounding that can exceed half a bf16 ulp
    by ~1e-8.)"""
    import gpu_helpers as gh
    from shifted_window_attention_pad_b200 import WORKLOADS
    from shifted_window_attention_pad_b200.synth import make_inputs, as_f64
    wl = WORKLOADS["ragged-90x180-w8"]
    inp = make_inputs(wl)
    s = oracle.make_shape(wl.B, wl.H, wl.W, wl.win, wl.shift, wl.heads, wl.head_dim)
    o, _ = oracle.forward(s, *(as_f64(inp[n]) for n in ("q", "k", "v", "table")), want_lse=False)
    rounded = torch.from_numpy(o).to(torch.bfloat16).double().numpy()
    assert gh.err_bf16(rounded, o) < 1e-6
    assert gh.err_bf16(rounded, o, storage_rounding=False) > gh.BF16_TOL
    bad = rounded.copy()
    rms = np.sqrt(np.mean(o * o))
    bad.reshape(-1)[12345] += 0.03 * rms + gh.half_ulp_bf16(o.reshape(-1)[12345])
    assert gh.err_bf16(bad, o) > gh.BF16_TOL


# ---------------------------------------------------------------------------
# Valid extent (tokens that cover only padded field pixels, Table I): pins
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("H,W,valid,win,shift", [(16, 24, (13, 21), 8, 4), (10, 12, (9, 12), 4, 2),
                                                 (12, 8, (12, 7), (4, 4), (0, 2))])
def test_valid_extent_equals_the_smaller_grid_when_padding_agrees(H, W, valid, win, shift):
    """When the stored grid and its valid extent pad to the same window
    multiple, the tokens beyond the extent are exactly the pad tokens of the
    smaller grid: the valid region's outputs equal a plain run on the smaller
    grid, and every stored token beyond the extent gets exact zeros."""
    Hv, Wv = valid
    heads, hd = 2, 3
    s, q, k, v, T, do = problem(1, H, W, win, shift, heads, hd, seed=61)
    sv = oracle.make_shape(1, H, W, win, shift, heads, hd, valid=valid)
    assert oracle.padded_hw(sv) == oracle.padded_hw(oracle.make_shape(1, Hv, Wv, win, shift,
                                                                      heads, hd))
    o, lse = oracle.forward(sv, q, k, v, T)
    dq, dk, dv, dT = oracle.backward(sv, q, k, v, T, do)
    ss = oracle.make_shape(1, Hv, Wv, win, shift, heads, hd)
    cut = lambda a: np.ascontiguousarray(a[:, :Hv, :Wv])
    o2, lse2 = oracle.forward(ss, cut(q), cut(k), cut(v), T)
    dq2, dk2, dv2, dT2 = oracle.backward(ss, cut(q), cut(k), cut(v), T, cut(do))
    for a, b in ((o, o2), (lse, lse2), (dq, dq2), (dk, dk2), (dv, dv2)):
        np.testing.assert_allclose(a[:, :Hv, :Wv], b, rtol=0, atol=1e-13)
        outside = np.ones(a.shape[:3], bool)
        outside[:, :Hv, :Wv] = False
        assert np.all(a[outside] == 0.0)
    np.testing.assert_allclose(dT, dT2, rtol=0, atol=1e-12)


def test_data_beyond_the_valid_extent_changes_nothing():
    """Tokens beyond the valid extent are masked: new q, k, v, dO values there
    leave every output bit-identical."""
    heads, hd = 2, 4
    s, q, k, v, T, do = problem(1, 14, 19, 4, 2, heads, hd, seed=62)
    sv = oracle.make_shape(1, 14, 19, 4, 2, heads, hd, valid=(11, 15))
    ref_f = oracle.forward(sv, q, k, v, T)
    ref_b = oracle.backward(sv, q, k, v, T, do)
    q2, k2, v2, do2 = (a.copy() for a in (q, k, v, do))
    for a in (q2, k2, v2, do2):
        a[:, 11:] = 7.0
        a[:, :, 15:] = -3.0
    for a, b in zip(ref_f + ref_b, oracle.forward(sv, q2, k2, v2, T) +
                    oracle.backward(sv, q2, k2, v2, T, do2)):
        assert np.array_equal(a, b)


def test_index_map_marks_tokens_beyond_the_valid_extent_as_padding():
    s = oracle.make_shape(1, 9, 10, 4, 2, 1, 1)
    sv = oracle.make_shape(1, 9, 10, 4, 2, 1, 1, valid=(7, 8))
    m, mv = oracle.index_map(s), oracle.index_map(sv)
    y, x = np.divmod(np.where(m >= 0, m, 0), 10)
    keep = (m >= 0) & (y < 7) & (x < 8)
    assert np.array_equal(mv, np.where(keep, m, -1))
