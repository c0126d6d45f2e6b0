"""Head and batch partitions on two gloo ranks on the CPU.

Each rank runs the partition logic of shifted_window_attention_pad_b200.parallel
with the fp64 oracle standing in for the kernels (the CPU has no kernels);
the assembled outputs and the summed bias-table gradient must equal one
oracle run over the whole problem."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from shifted_window_attention_pad_b200 import binding as sb
from shifted_window_attention_pad_b200 import parallel as par

WORLD = 2


class OracleOps:
    """The fp64 oracle behind the Ops interface (CPU float64 tensors)."""

    @staticmethod
    def _shape(d):
        return oracle.Shape(d.B, d.H, d.W, d.win_h, d.win_w, d.shift_h, d.shift_w, d.heads,
                            d.head_dim, d.valid_h, d.valid_w)

    def forward(self, desc, q, k, v, table, want_lse=False):
        o, lse = oracle.forward(self._shape(desc), q.numpy(), k.numpy(), v.numpy(), table.numpy(),
                                want_lse=want_lse)
        o = torch.from_numpy(o)
        return (o, torch.from_numpy(lse)) if want_lse else o

    def backward(self, desc, q, k, v, table, dout):
        r = oracle.backward(self._shape(desc), q.numpy(), k.numpy(), v.numpy(), table.numpy(),
                            dout.numpy())
        return tuple(torch.from_numpy(a) for a in r)

    def backward_partial(self, desc, q, k, v, table, dout):
        dq, dk, dv, dT = self.backward(desc, q, k, v, table, dout)
        return dq, dk, dv, dT, None

    def finish(self, desc, partial, state):
        return partial

    # A row band from the oracle on the whole grid: the band's rows and its
    # halo rows at their places, zeros elsewhere. The band's windows see only
    # those rows, so their outputs are the band's. In the backward the band's
    # own first shift_h rows get dO = 0 (the band above owns their window
    # row), so no other window adds to the bias-table gradient.
    def _assemble(self, gd, y0, band, halo, zero_top=False):
        g = torch.zeros((band.shape[0], gd.H) + tuple(band.shape[2:]), dtype=band.dtype)
        hr = band.shape[1]
        g[:, y0:y0 + hr] = band
        if zero_top:
            g[:, y0:y0 + gd.shift_h] = 0
        hy = (y0 + hr) % gd.H
        g[:, hy:hy + gd.shift_h] = halo
        return g, hy

    def forward_band(self, gd, desc, y0, interior, q, k, v, hq, hk, hv, table, want_lse):
        (Q, hy), (K, _), (V, _) = (self._assemble(gd, y0, a, b) for a, b in
                                   ((q, hq), (k, hk), (v, hv)))
        o, lse = self.forward(gd, Q, K, V, table, want_lse=True)
        hr, s = q.shape[1], gd.shift_h
        res = (o[:, y0:y0 + hr].clone(), o[:, hy:hy + s].clone())
        return res + (lse[:, y0:y0 + hr].clone(), lse[:, hy:hy + s].clone()) if want_lse else res

    def backward_band(self, gd, desc, y0, interior, q, k, v, dout, hq, hk, hv, hdo, table):
        (Q, hy), (K, _), (V, _) = (self._assemble(gd, y0, a, b) for a, b in
                                   ((q, hq), (k, hk), (v, hv)))
        DO, _ = self._assemble(gd, y0, dout, hdo, zero_top=True)
        dq, dk, dv, dT = self.backward(gd, Q, K, V, table, DO)
        hr, s = q.shape[1], gd.shift_h
        band = [a[:, y0:y0 + hr].clone() for a in (dq, dk, dv)]
        halo = [a[:, hy:hy + s].clone() for a in (dq, dk, dv)]
        return (*band, *halo, dT, None)


def _inputs(B, H, W, heads, hd, win, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    shape = (B, H, W, heads, hd)
    q, k, v, do = (torch.from_numpy(rng.standard_normal(shape)) for _ in range(4))
    T = torch.from_numpy(rng.standard_normal(((2 * win - 1) ** 2, heads)) * 0.02)
    return q, k, v, T, do


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, kind, out, world=WORLD):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ops = OracleOps()
        g = par.Group.current()
        desc = sb.make_desc(3, 20, 28, 8, 4, 3, 16, "f32")
        q, k, v, T, do = _inputs(3, 20, 28, 3, 16, 8, 5)
        if kind == "rows":
            desc = sb.make_desc(2, 45, 28, 8, 4, 2, 16, "f32")   # 45 rows: padded last band
            q, k, v, T, do = _inputs(2, 45, 28, 2, 16, 8, 6)
            ld, y0, y1, _ = par.band_shard(desc, world, rank)
            sl = lambda t: t[:, y0:y1].contiguous()
            o, lse = par.forward_rows(desc, sl(q), sl(k), sl(v), T, want_lse=True, ops=ops)
            dq, dk, dv, dT = par.backward_rows(desc, sl(q), sl(k), sl(v), T, sl(do), g=g, ops=ops)
            res = dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv, dT=dT, lo=y0, hi=y1)
        elif kind == "heads":
            ld, h0, h1 = par.head_shard(desc, WORLD, rank)
            sl = lambda t: t[:, :, :, h0:h1].contiguous()
            o = par.forward_heads(ld, sl(q), sl(k), sl(v), T[:, h0:h1].contiguous(), ops=ops)
            dq, dk, dv, dT = par.backward_heads(ld, sl(q), sl(k), sl(v), T[:, h0:h1].contiguous(),
                                                sl(do), ops=ops)
            dT_all = par.gather_heads(dT, desc, g)
            res = dict(o=o, dq=dq, dk=dk, dv=dv, dT=dT_all, lo=h0, hi=h1)
        else:
            ld, b0, b1 = par.batch_shard(desc, WORLD, rank)
            sl = lambda t: t[b0:b1].contiguous()
            o = par.forward_batch(ld, sl(q), sl(k), sl(v), T, ops=ops)
            dq, dk, dv, dT = par.backward_batch(ld, sl(q), sl(k), sl(v), T, sl(do), g=g, ops=ops)
            res = dict(o=o, dq=dq, dk=dk, dv=dv, dT=dT, lo=b0, hi=b1)
        torch.save(res, os.path.join(out, "rank%d.pt" % rank))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("kind", ["heads", "batch"])
def test_partition_on_two_gloo_ranks_matches_one_run(kind, tmp_path):
    mp.start_processes(_worker, args=(_free_port(), kind, str(tmp_path)), nprocs=WORLD,
                       start_method="spawn", join=True)
    q, k, v, T, do = _inputs(3, 20, 28, 3, 16, 8, 5)
    s = oracle.Shape(3, 20, 28, 8, 8, 4, 4, 3, 16)
    o, _ = oracle.forward(s, q.numpy(), k.numpy(), v.numpy(), T.numpy(), want_lse=False)
    dq, dk, dv, dT = oracle.backward(s, q.numpy(), k.numpy(), v.numpy(), T.numpy(), do.numpy())
    full = dict(o=o, dq=dq, dk=dk, dv=dv)
    for r in range(WORLD):
        res = torch.load(os.path.join(str(tmp_path), "rank%d.pt" % r))
        lo, hi = res["lo"], res["hi"]
        for n, ref in full.items():
            part = ref[:, :, :, lo:hi] if kind == "heads" else ref[lo:hi]
            np.testing.assert_allclose(res[n].numpy(), part, rtol=0, atol=1e-12)
        # every rank ends with the whole table: gathered heads, or summed images
        np.testing.assert_allclose(res["dT"].numpy(), dT, rtol=0,
                                   atol=1e-12 * max(1.0, np.abs(dT).max()))


def test_split_range_covers_every_index_once():
    for n in (1, 2, 3, 7, 16, 33):
        for world in range(1, min(n, 9) + 1):
            idx = [i for r in range(world) for i in range(*par.split_range(n, world, r))]
            assert idx == list(range(n))
    with pytest.raises(ValueError):
        par.head_shard(sb.make_desc(1, 8, 8, 8, 0, 2, 16, "f32"), 3, 2)


@pytest.mark.parametrize("world", [2, 3])
def test_row_bands_with_boundary_exchange_match_one_run(world, tmp_path):
    """Rows split into bands over gloo ranks: only shift_h boundary rows move
    (inputs up, outputs down), the bias-table gradient is summed over bands,
    and the assembled result equals one oracle run over the whole grid."""
    mp.start_processes(_worker, args=(_free_port(), "rows", str(tmp_path), world), nprocs=world,
                       start_method="spawn", join=True)
    q, k, v, T, do = _inputs(2, 45, 28, 2, 16, 8, 6)
    s = oracle.Shape(2, 45, 28, 8, 8, 4, 4, 2, 16)
    o, lse = oracle.forward(s, q.numpy(), k.numpy(), v.numpy(), T.numpy())
    dq, dk, dv, dT = oracle.backward(s, q.numpy(), k.numpy(), v.numpy(), T.numpy(), do.numpy())
    rows = set()
    for r in range(world):
        res = torch.load(os.path.join(str(tmp_path), "rank%d.pt" % r))
        lo, hi = res["lo"], res["hi"]
        rows |= set(range(lo, hi))
        for n, ref in dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv).items():
            np.testing.assert_allclose(res[n].numpy(), ref[:, lo:hi], rtol=0, atol=1e-12,
                                       err_msg="%s rank %d" % (n, r))
        np.testing.assert_allclose(res["dT"].numpy(), dT, rtol=0,
                                   atol=1e-12 * max(1.0, np.abs(dT).max()))
    assert rows == set(range(45))
