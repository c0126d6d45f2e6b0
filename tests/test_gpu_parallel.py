"""The head and batch partitions on one GPU, shard after shard (no rank waits
on another): every shard's outputs equal the matching slice of one call over
the whole problem, bit for bit, and the exact bias-gradient sums of the batch
shards, added as int64 words and converted once, give the whole batch's
bias-table gradient bit for bit."""
import numpy as np
import pytest
import torch

from shifted_window_attention_pad_b200 import binding as sb
from shifted_window_attention_pad_b200 import parallel as par
from shifted_window_attention_pad_b200.synth import make_inputs
from shifted_window_attention_pad_b200.workloads import Workload

pytestmark = pytest.mark.gpu

# (B, H, W, window, shift, heads, head_dim, seed, path)
CASES = [(3, 36, 44, 8, 4, 5, 64, 51, 1), (2, 40, 52, 16, 8, 3, 64, 52, 3),
         (2, 64, 64, 32, 16, 3, 128, 53, 4)]


@pytest.fixture(scope="module", autouse=True)
def _built():
    from shifted_window_attention_pad_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _setup(case):
    B, H, W, win, shift, heads, hd, seed, path = case
    wl = Workload("par", B, H, W, win, shift, heads, hd, "bf16", seed)
    inp = {n: t.cuda() for n, t in make_inputs(wl).items()}
    d = sb.desc_for(wl)
    assert sb.swin_wattn_path(d) == path
    return d, inp


@pytest.mark.parametrize("case", CASES, ids=lambda c: "path%d" % c[-1])
@pytest.mark.parametrize("world", [2, 3])
def test_head_shards_equal_the_whole_call(case, world):
    d, inp = _setup(case)
    q, k, v, T, do = (inp[n] for n in ("q", "k", "v", "table", "dout"))
    o = sb.forward(d, q, k, v, T)
    dq, dk, dv, dT = sb.backward(d, q, k, v, T, do)
    for r in range(world):
        ld, h0, h1 = par.head_shard(d, world, r)
        sl = lambda t: t[:, :, :, h0:h1].contiguous()
        Tl = T[:, h0:h1].contiguous()
        assert torch.equal(par.forward_heads(ld, sl(q), sl(k), sl(v), Tl), sl(o))
        g = par.backward_heads(ld, sl(q), sl(k), sl(v), Tl, sl(do))
        for got, want in zip(g[:3], (dq, dk, dv)):
            assert torch.equal(got, sl(want))
        assert torch.equal(g[3], dT[:, h0:h1])


@pytest.mark.parametrize("case", CASES, ids=lambda c: "path%d" % c[-1])
def test_batch_shards_with_summed_exact_sums_equal_the_whole_batch(case):
    d, inp = _setup(case)
    q, k, v, T, do = (inp[n] for n in ("q", "k", "v", "table", "dout"))
    dq, dk, dv, dT = sb.backward(d, q, k, v, T, do)
    ops = par.LIBRARY
    total, state = None, None
    for r in range(d.B):                       # one image per simulated rank
        ld, b0, b1 = par.batch_shard(d, d.B, r)
        sl = lambda t: t[b0:b1].contiguous()
        gq, gk, gv, partial, st = ops.backward_partial(ld, sl(q), sl(k), sl(v), T, sl(do))
        for got, want in zip((gq, gk, gv), (dq, dk, dv)):
            assert torch.equal(got, sl(want))
        if total is None:
            total, state = partial.clone(), st
        else:
            total += partial                   # what a SUM all-reduce of the words does
    state_view = sb.dbias_sums_view(par.batch_shard(d, d.B, 0)[0], state)
    state_view.copy_(total)
    got = ops.finish(par.batch_shard(d, d.B, 0)[0], state_view, state)
    torch.cuda.synchronize()
    assert torch.equal(got, dT)
    assert np.isfinite(got.cpu().numpy()).all()


# (B, H, W, heads, head_dim, seed, world): a ragged last band (45 rows, padded
# to 48) and the 1/12-degree token grid on four bands
BANDS = [(2, 45, 44, 3, 64, 61, 1), (2, 45, 44, 3, 64, 61, 2), (2, 45, 44, 3, 32, 62, 3),
         (1, 256, 544, 4, 64, 63, 4), (1, 40, 36, 2, 128, 64, 2)]


@pytest.mark.parametrize("case", BANDS, ids=lambda c: "%dx%d-hd%d-bands%d" % (c[1], c[2], c[4], c[6]))
def test_row_bands_reassemble_the_whole_grid_bit_for_bit(case):
    """Each band's kernels read the shift_h rows below the band from a halo
    tensor and write those rows' outputs to a halo output; the band's own
    first shift_h rows come from the band above. Put back together (and the
    exact bias-gradient sums added over bands), the bands give the whole-grid
    call's bits."""
    B, H, W, heads, hd, seed, world = case
    wl = Workload("bands", B, H, W, 8, 4, heads, hd, "bf16", seed)
    d = sb.desc_for(wl)
    assert sb.swin_wattn_path(d) == 1
    inp = {n: t.cuda() for n, t in make_inputs(wl).items()}
    q, k, v, T, do = (inp[n] for n in ("q", "k", "v", "table", "dout"))
    o, lse = sb.forward(d, q, k, v, T, want_lse=True)
    dq, dk, dv, dT = sb.backward(d, q, k, v, T, do)
    s = d.shift_h
    got = {n: torch.full_like(t, float("nan")) for n, t in
           dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv).items()}
    ops = par.LIBRARY
    total, state, last_desc = None, None, None
    for r in range(world):
        ld, y0, y1, interior = par.band_shard(d, world, r)
        hy = y1 % H
        band = lambda t: t[:, y0:y1].contiguous()
        halo = lambda t: t[:, hy:hy + s].contiguous()
        fo, fo_h, fl, fl_h = ops.forward_band(d, ld, y0, interior, band(q), band(k), band(v),
                                              halo(q), halo(k), halo(v), T, True)
        res = ops.backward_band(d, ld, y0, interior, band(q), band(k), band(v), band(do), halo(q),
                                halo(k), halo(v), halo(do), T)
        for n, a, ah in (("o", fo, fo_h), ("lse", fl, fl_h), ("dq", res[0], res[3]),
                         ("dk", res[1], res[4]), ("dv", res[2], res[5])):
            got[n][:, y0 + s:y1] = a[:, s:]
            got[n][:, hy:hy + s] = ah
        total = res[6].clone() if total is None else total + res[6]
        state, last_desc = res[7], ld
    sb.dbias_sums_view(last_desc, state).copy_(total)
    dT_bands = ops.finish(last_desc, sb.dbias_sums_view(last_desc, state), state)
    torch.cuda.synchronize()
    for n, want in dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv).items():
        assert torch.equal(got[n], want), n
    assert torch.equal(dT_bands, dT)
