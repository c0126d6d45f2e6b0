"""Multi-GPU partitions of shifted-window attention: one process per GPU,
torch.distributed (NCCL on GPUs) for the plumbing, the library's kernels for
every step of the computation.

Windows, heads and batch images are independent once the shifted layout is
fixed (TERRA page, Abstract: windows are the unit of "shifted-window
execution"; Fig. 6 and Table III place window layouts on devices), so the op
itself needs no exchange in the head and batch partitions:

* heads: rank r owns a contiguous range of heads (the layout a head-sharded
  QKV projection produces): its q, k, v, dO are [B, H, W, heads_r, hd] and its
  slice of the bias table [bins, heads_r]. Nothing crosses ranks; each rank's
  bias-table gradient covers its own heads (``gather_heads`` assembles the
  whole table where a caller wants it).
* batch: rank r owns images [b0, b1) of the batch and the whole bias table.
  The bias-table gradient is the sum over all images, hence over ranks. The
  tensor-core kernels keep it as exact integer sums (the library's
  SWIN_FLAG_DBIAS_SUMS); ranks add those int64 words with one all-reduce and
  convert once, so every rank gets the bits one GPU would give for the whole
  batch, whatever the reduction order.

The compute is an ``Ops`` object: ``LibraryOps`` (the CUDA library, the only
one the package provides) by default. Tests on CPU ranks pass their own.
"""
from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import binding as sb


def split_range(n, world, rank):
    """Contiguous near-even split of range(n): (lo, hi) of `rank`."""
    if not 0 <= rank < world:
        raise ValueError("rank %d outside a world of %d" % (rank, world))
    q, r = divmod(n, world)
    lo = rank * q + min(rank, r)
    return lo, lo + q + (1 if rank < r else 0)


def _desc_with(desc, **kw):
    fields = {n: getattr(desc, n) for n, _ in desc._fields_}
    fields.update(kw)
    return sb.SwinWattnDesc(**fields)


def head_shard(desc, world, rank):
    """(local description, h0, h1) of rank `rank` in a head partition."""
    h0, h1 = split_range(desc.heads, world, rank)
    if h1 <= h0:
        raise ValueError("more ranks (%d) than heads (%d)" % (world, desc.heads))
    return _desc_with(desc, heads=h1 - h0), h0, h1


def batch_shard(desc, world, rank):
    """(local description, b0, b1) of rank `rank` in a batch partition."""
    b0, b1 = split_range(desc.B, world, rank)
    if b1 <= b0:
        raise ValueError("more ranks (%d) than images (%d)" % (world, desc.B))
    return _desc_with(desc, B=b1 - b0), b0, b1


class LibraryOps:
    """The library's kernels through the binding (device tensors)."""

    def forward(self, desc, q, k, v, table, want_lse=False):
        return sb.forward(desc, q, k, v, table, want_lse=want_lse)

    def backward(self, desc, q, k, v, table, dout):
        return sb.backward(desc, q, k, v, table, dout)

    def backward_partial(self, desc, q, k, v, table, dout):
        """(dq, dk, dv, partial, state): `partial` is what ranks add up with
        one SUM all-reduce, `finish(desc, partial, state)` turns the added
        words into the bias-table gradient."""
        if sb.swin_wattn_path(desc) == 0:       # portable kernels: fp32 partials
            dq, dk, dv, dT = sb.backward(desc, q, k, v, table, dout)
            return dq, dk, dv, dT, None
        d = _desc_with(desc, flags=desc.flags | sb.SWIN_FLAG_DBIAS_SUMS)
        ws = sb.new_workspace(d, q.device)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        sb.swin_wattn_bwd(d, q, k, v, table, dout, dq, dk, dv, None, ws)
        return dq, dk, dv, sb.dbias_sums_view(d, ws), ws

    def forward_band(self, gdesc, desc, y0, interior, q, k, v, hq, hk, hv, table, want_lse):
        """(out, out_halo[, lse, lse_halo]) of one row band."""
        out, out_h = torch.empty_like(q), torch.empty_like(hq)
        lse = lse_h = None
        if want_lse:
            lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
            lse_h = torch.empty(hq.shape[:-1], dtype=torch.float32, device=q.device)
        halo = sb.make_halo(interior, q=hq, k=hk, v=hv, out=out_h, lse=lse_h)
        sb.swin_wattn_fwd_band(desc, halo, q, k, v, table, out, lse)
        return (out, out_h, lse, lse_h) if want_lse else (out, out_h)

    def backward_band(self, gdesc, desc, y0, interior, q, k, v, dout, hq, hk, hv, hdo, table):
        """(dq, dk, dv, dq_halo, dk_halo, dv_halo, partial, state) of one row
        band; `partial` adds over bands like backward_partial's."""
        d = _desc_with(desc, flags=desc.flags | sb.SWIN_FLAG_DBIAS_SUMS)
        ws = sb.new_workspace(d, q.device)
        g = [torch.empty_like(t) for t in (q, k, v, hq, hk, hv)]
        halo = sb.make_halo(interior, q=hq, k=hk, v=hv, dout=hdo, dq=g[3], dk=g[4], dv=g[5])
        sb.swin_wattn_bwd_band(d, halo, q, k, v, table, dout, g[0], g[1], g[2], None, ws)
        return (*g, sb.dbias_sums_view(d, ws), ws)

    def finish(self, desc, partial, state):
        if state is None:
            return partial
        dT = torch.empty((_bins(desc), desc.heads), dtype=torch.float32, device=partial.device)
        return sb.swin_wattn_dbias_finish(desc, state, dT)


def _bins(desc):
    return (2 * desc.win_h - 1) * (2 * desc.win_w - 1)


LIBRARY = LibraryOps()


@dataclass
class Group:
    """Rank, world size and process group (None = the default group)."""
    rank: int
    world: int
    group: object = None

    @staticmethod
    def current(group=None):
        if dist.is_available() and dist.is_initialized():
            return Group(dist.get_rank(group), dist.get_world_size(group), group)
        return Group(0, 1, None)


# ---- head partition -------------------------------------------------------------
def forward_heads(desc, q, k, v, table_local, want_lse=False, ops=None):
    """Forward of this rank's heads; q, k, v hold only them. No exchange."""
    return (ops or LIBRARY).forward(desc, q, k, v, table_local, want_lse=want_lse)


def backward_heads(desc, q, k, v, table_local, dout, ops=None):
    """Backward of this rank's heads: dq, dk, dv and the bias-table gradient
    rows [bins, heads_r] of its own heads. No exchange."""
    return (ops or LIBRARY).backward(desc, q, k, v, table_local, dout)


def gather_heads(dT_local, world_desc, g=None):
    """The whole [bins, heads] bias-table gradient on every rank, from each
    rank's [bins, heads_r] slice (one all-gather)."""
    g = g or Group.current()
    if g.world == 1:
        return dT_local
    shapes = [split_range(world_desc.heads, g.world, r) for r in range(g.world)]
    bufs = [torch.empty((dT_local.shape[0], h1 - h0), dtype=dT_local.dtype,
                        device=dT_local.device) for (h0, h1) in shapes]
    if len({b.shape for b in bufs}) == 1:
        dist.all_gather(bufs, dT_local.contiguous(), group=g.group)
    else:   # uneven head counts: pad to the largest slice
        wmax = max(b.shape[1] for b in bufs)
        pad = torch.zeros((dT_local.shape[0], wmax), dtype=dT_local.dtype, device=dT_local.device)
        pad[:, :dT_local.shape[1]] = dT_local
        full = [torch.empty_like(pad) for _ in range(g.world)]
        dist.all_gather(full, pad, group=g.group)
        bufs = [f[:, :b.shape[1]] for f, b in zip(full, bufs)]
    return torch.cat(bufs, dim=1)


# ---- batch partition ----------------------------------------------------------------
def forward_batch(desc, q, k, v, table, want_lse=False, ops=None):
    """Forward of this rank's images; no exchange."""
    return (ops or LIBRARY).forward(desc, q, k, v, table, want_lse=want_lse)


def backward_batch(desc, q, k, v, table, dout, g=None, ops=None):
    """Backward of this rank's images; the bias-table gradient is summed over
    all ranks (one all-reduce of the exact sums, converted once), so every
    rank returns the same table."""
    ops = ops or LIBRARY
    g = g or Group.current()
    dq, dk, dv, partial, state = ops.backward_partial(desc, q, k, v, table, dout)
    if g.world > 1:
        dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=g.group)
    return dq, dk, dv, ops.finish(desc, partial, state)


# ---- row bands (window strips) ------------------------------------------------------
# Rank r owns rows [y0, y1) of the token grid, bands of whole window rows (the
# last band takes what is left, padding included). With the shift, the last
# window row of a band reads the shift_h rows below the band, which the next
# rank owns (the last rank reads the grid's first rows: the wrap), and its
# outputs for those rows belong to that rank. So each step exchanges only
# boundary rows: shift_h rows of every input go up to the previous rank, the
# outputs of shift_h rows come back down (TERRA page, Table III:
# "Boundary-only P2P"); the bias-table gradient is summed over bands like
# over batch shards.
def band_rows(H, win_h, world, rank):
    """(y0, y1) of `rank`: bands of ceil(window rows / world) window rows."""
    n_wy = -(-H // win_h)
    per = -(-n_wy // world) * win_h
    y0, y1 = rank * per, min((rank + 1) * per, H)
    if y1 <= y0:
        raise ValueError("%d ranks leave rank %d no rows of a %d-row grid" % (world, rank, H))
    return y0, y1


def band_shard(desc, world, rank):
    """(local description, y0, y1, interior) of rank `rank` in a row partition."""
    y0, y1 = band_rows(desc.H, desc.win_h, world, rank)
    if y1 - y0 < desc.shift_h:
        raise ValueError("band of %d rows is thinner than the shift %d" % (y1 - y0, desc.shift_h))
    vh = 0
    if desc.valid_h:
        if desc.valid_h < y0 + 1:
            raise ValueError("a band without valid rows")
        vh = min(desc.valid_h, y1) - y0
    return _desc_with(desc, H=y1 - y0, valid_h=vh), y0, y1, rank != world - 1


def _rows(t, n):
    return t[:, :n].contiguous()


def _exchange(send, recv_like, to, frm, g):
    """Sends tensors `send` to rank `to` and returns tensors shaped like
    `recv_like` received from rank `frm` (one batch of peer-to-peer ops)."""
    if g.world == 1:
        return [t.clone() for t in send]
    bufs = [torch.empty_like(t) for t in recv_like]
    ops = [dist.P2POp(dist.isend, t, to, group=g.group) for t in send]
    ops += [dist.P2POp(dist.irecv, b, frm, group=g.group) for b in bufs]
    for w in dist.batch_isend_irecv(ops):
        w.wait()
    return bufs


def forward_rows(desc, q, k, v, table, want_lse=False, g=None, ops=None):
    """Forward of this rank's band; q, k, v are its rows [B, y1-y0, W, heads, hd].
    Returns out (and lse) for the band's rows."""
    ops = ops or LIBRARY
    g = g or Group.current()
    ld, y0, y1, interior = band_shard(desc, g.world, g.rank)
    s = desc.shift_h
    up, down = (g.rank - 1) % g.world, (g.rank + 1) % g.world
    mine = [_rows(t, s) for t in (q, k, v)]
    hq, hk, hv = _exchange(mine, mine, up, down, g)
    res = ops.forward_band(desc, ld, y0, interior, q, k, v, hq, hk, hv, table, want_lse)
    out, out_h = res[0], res[1]
    back = [out_h] + ([res[3]] if want_lse else [])
    like = [_rows(out, s)] + ([_rows(res[2], s)] if want_lse else [])
    got = _exchange(back, like, down, up, g)
    out[:, :s] = got[0]
    if want_lse:
        res[2][:, :s] = got[1]
        return out, res[2]
    return out


def backward_rows(desc, q, k, v, table, dout, g=None, ops=None):
    """Backward of this rank's band: dq, dk, dv of its rows and the
    bias-table gradient of the whole grid (summed over bands, exactly)."""
    ops = ops or LIBRARY
    g = g or Group.current()
    ld, y0, y1, interior = band_shard(desc, g.world, g.rank)
    s = desc.shift_h
    up, down = (g.rank - 1) % g.world, (g.rank + 1) % g.world
    mine = [_rows(t, s) for t in (q, k, v, dout)]
    hq, hk, hv, hdo = _exchange(mine, mine, up, down, g)
    dq, dk, dv, dq_h, dk_h, dv_h, partial, state = ops.backward_band(
        desc, ld, y0, interior, q, k, v, dout, hq, hk, hv, hdo, table)
    got = _exchange([dq_h, dk_h, dv_h], [_rows(dq, s), _rows(dk, s), _rows(dv, s)], down, up, g)
    dq[:, :s], dk[:, :s], dv[:, :s] = got
    if g.world > 1:
        dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=g.group)
    return dq, dk, dv, ops.finish(ld, partial, state)
