"""Sequence-parallel routing of the hybrid attention layer over several GPUs.

The pages run the layer with Ulysses sequence parallelism (project page,
"Parallelization & Few-Step Generation"): outside the attention the tokens are
sharded along the sequence, one contiguous token range per GPU; an all-to-all
turns that into a head shard (every GPU gets all tokens of some heads), the
attention runs per head, and a reverse all-to-all returns the output to the
token shard. Every (batch, head) pair of this op is independent in both
branches, so the head shard needs no other exchange. Two routings:

  ulysses_hybrid_fwd       plain Ulysses: every GPU runs both branches (the
                           whole vdn_hybrid_attn_fwd) on H / N heads.
  branch_split_hybrid_fwd  the pages' branch-specialised split: an uneven
                           all-to-all sends q, k, v of each head to one
                           "softmax" GPU and q, k, v, beta to one "linear"
                           GPU (the pages use 5 + 3 of 8 B200s); the softmax
                           GPUs run vdn_window_softmax_fwd_f32out, the linear
                           GPUs vdn_vda_scan_fwd_f32out, and a reverse uneven
                           all-to-all returns o_soft and o_lin (float32) to
                           the token shards, which finish with
                           vdn_gated_combine_fwd using the gates they hold
                           (the gates never move).

The text tokens (keys, values, write strengths) are small and replicated on
every GPU; each head worker takes its heads' slice.

This module only moves data: packing the per-destination slices, one
all_to_all_single over bytes per exchange (NCCL on GPUs), and unpacking. The
per-head computation is done by the library's entry points; the ``compute``
arguments exist so that the routing can be exercised on CPU processes (gloo)
with another implementation of the same entry points.
"""

from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Callable, Dict, List, Optional, Sequence

import torch
import torch.distributed as dist

from .synth import Layout


# ------------------------------------------------------------------ planning

def even_ranges(total: int, parts: int) -> List[range]:
    """total items in `parts` contiguous ranges whose sizes differ by at most one."""
    return [range(total * p // parts, total * (p + 1) // parts) for p in range(parts)]


@dataclass(frozen=True)
class Plan:
    """Who holds what. tokens[r]: the token range of rank r's sequence shard.
    soft_heads[r] / lin_heads[r]: heads whose softmax / linear branch rank r
    computes (empty when rank r does no such work)."""
    world: int
    tokens: List[range]
    soft_heads: List[range]
    lin_heads: List[range]


def ulysses_plan(layout: Layout, world: int) -> Plan:
    """Plain Ulysses: rank r holds tokens [L r / N, L (r+1) / N) and computes
    both branches of heads [H r / N, H (r+1) / N)."""
    if layout.H < world:
        raise ValueError(f"{layout.H} heads cannot be spread over {world} ranks")
    heads = even_ranges(layout.H, world)
    return Plan(world, even_ranges(layout.L, world), heads, heads)


def branch_split_plan(layout: Layout, world: int, n_soft: int) -> Plan:
    """Branch-specialised: ranks 0 .. n_soft-1 compute the softmax branch of
    H / n_soft heads each, ranks n_soft .. N-1 the linear branch of
    H / (N - n_soft) heads each; every rank holds a token shard."""
    n_lin = world - n_soft
    if n_soft < 1 or n_lin < 1:
        raise ValueError("both branches need at least one rank")
    if layout.H < max(n_soft, n_lin):
        raise ValueError(f"{layout.H} heads cannot be spread over {max(n_soft, n_lin)} ranks")
    empty = range(0, 0)
    sh = even_ranges(layout.H, n_soft)
    lh = even_ranges(layout.H, n_lin)
    soft = [sh[r] if r < n_soft else empty for r in range(world)]
    lin = [lh[r - n_soft] if r >= n_soft else empty for r in range(world)]
    return Plan(world, even_ranges(layout.L, world), soft, lin)


# ------------------------------------------------------------------ exchange

def _flat_bytes(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().view(-1).view(torch.uint8)


def exchange(send: Sequence[Sequence[torch.Tensor]], recv_specs: Sequence[Sequence[tuple]],
             device, group=None) -> List[List[torch.Tensor]]:
    """One all_to_all_single over bytes. send[p]: the tensors this rank sends to
    rank p (any dtypes); recv_specs[p]: (shape, dtype) of each tensor it gets
    from rank p, in the order p sends them. Both sides derive the sizes from
    the same plan, so no sizes are exchanged. Returns the received tensors."""
    world = len(send)
    in_parts = [[_flat_bytes(t) for t in ts] for ts in send]
    in_sizes = [sum(int(b.numel()) for b in bs) for bs in in_parts]
    out_sizes = [sum(int(torch.Size(s).numel()) * torch.empty((), dtype=dt).element_size()
                     for s, dt in specs) for specs in recv_specs]
    flat_in = [b for bs in in_parts for b in bs]
    send_buf = torch.cat(flat_in) if flat_in else torch.empty(0, dtype=torch.uint8, device=device)
    recv_buf = torch.empty(sum(out_sizes), dtype=torch.uint8, device=device)
    if world > 1:
        dist.all_to_all_single(recv_buf, send_buf.to(device), output_split_sizes=out_sizes,
                               input_split_sizes=in_sizes, group=group)
    else:
        recv_buf.copy_(send_buf)
    out, off = [], 0
    for specs in recv_specs:
        got = []
        for shape, dt in specs:
            n = int(torch.Size(shape).numel()) * torch.empty((), dtype=dt).element_size()
            got.append(recv_buf[off:off + n].view(dt).view(shape))
            off += n
        out.append(got)
    return out


def _heads(t: torch.Tensor, hr: range) -> torch.Tensor:
    """t[:, :, heads] of a [B, rows, H, ...] tensor (a copy, contiguous)."""
    return t[:, :, hr.start:hr.stop].contiguous()


def _assemble(pieces: Sequence[torch.Tensor], plan: Plan, B: int, L: int, h: int, tail, dtype,
              device) -> torch.Tensor:
    """[B, L, h, *tail] from the token-shard pieces [B, |tokens[p]|, h, *tail]."""
    full = torch.empty((B, L, h, *tail), dtype=dtype, device=device)
    for p, piece in enumerate(pieces):
        tr = plan.tokens[p]
        full[:, tr.start:tr.stop] = piece
    return full


def _scatter_heads(pieces: Dict[int, torch.Tensor], heads: Sequence[range], out: torch.Tensor):
    """out[:, :, heads[p]] = pieces[p] for the ranks that sent a piece."""
    for p, piece in pieces.items():
        hr = heads[p]
        out[:, :, hr.start:hr.stop] = piece


def _layout_heads(layout: Layout, h: int) -> Layout:
    return replace(layout, H=h)


# --------------------------------------------------------------- routings

@dataclass
class Shard:
    """One rank's token shard of the layer input: video tensors [B, |tokens|, H, d]
    (beta [B, |tokens|, H] float32), and the replicated text tensors."""
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    beta: torch.Tensor
    g_s: torch.Tensor
    g_l: torch.Tensor
    k_text: Optional[torch.Tensor]
    v_text: Optional[torch.Tensor]
    beta_text: Optional[torch.Tensor]


def _default_hybrid(layout, q, k, v, kt, vt, beta, bt, gs, gl, rms_weight, rms_eps):
    from . import vdn
    return vdn.hybrid_attn_fwd(layout, q, k, v, kt, vt, beta, bt, gs, gl, rms_weight=rms_weight,
                               rms_eps=rms_eps)


def _default_softmax(layout, q, k, v, kt, vt):
    from . import vdn
    return vdn.window_softmax_fwd(layout, q, k, v, kt, vt, out_f32=True)


def _default_linear(layout, q, k, v, kt, vt, beta, bt):
    from . import vdn
    return vdn.vda_scan_fwd(layout, q, k, v, kt, vt, beta, bt, out_f32=True)


def _default_combine(o_soft, o_lin, gs, gl, rms_weight, rms_eps):
    from . import vdn
    return vdn.gated_combine_fwd(o_soft, o_lin, gs, gl, rms_weight=rms_weight, rms_eps=rms_eps)


def _text(t, hr):
    return None if t is None else _heads(t, hr)


def ulysses_hybrid_fwd(layout: Layout, shard: Shard, rank: int, plan: Plan, group=None,
                       rms_weight=None, rms_eps: float = 1e-6,
                       hybrid: Callable = _default_hybrid) -> torch.Tensor:
    """Plain Ulysses over the ranks of `group`: returns this rank's token shard
    of the hybrid output, [B, |tokens[rank]|, H, d]."""
    B, H, d, L = layout.B, layout.H, layout.d, layout.L
    dev, dt, bt = shard.q.device, shard.q.dtype, shard.beta.dtype
    W = plan.world
    my_h = plan.soft_heads[rank]
    # token shard -> head shard: q, k, v, g_s, g_l and beta of each rank's heads
    send = [[_heads(t, plan.soft_heads[p]) for t in (shard.q, shard.k, shard.v, shard.g_s, shard.g_l,
                                                     shard.beta)] for p in range(W)]
    specs = []
    for p in range(W):
        n = len(plan.tokens[p])
        specs.append([((B, n, len(my_h), d), dt)] * 5 + [((B, n, len(my_h)), bt)])
    got = exchange(send, specs, dev, group)
    full = [_assemble([g[i] for g in got], plan, B, L, len(my_h), (d,) if i < 5 else (),
                      dt if i < 5 else bt, dev) for i in range(6)]
    q, k, v, gs, gl, beta = full
    out_h = hybrid(_layout_heads(layout, len(my_h)), q, k, v, _text(shard.k_text, my_h),
                   _text(shard.v_text, my_h), beta, _text(shard.beta_text, my_h), gs, gl,
                   rms_weight, rms_eps)
    # head shard -> token shard
    back = [[out_h[:, plan.tokens[p].start:plan.tokens[p].stop].contiguous()] for p in range(W)]
    n_mine = len(plan.tokens[rank])
    specs = [[((B, n_mine, len(plan.soft_heads[p]), d), dt)] for p in range(W)]
    got = exchange(back, specs, dev, group)
    out = torch.empty((B, n_mine, H, d), dtype=dt, device=dev)
    _scatter_heads({p: got[p][0] for p in range(W)}, plan.soft_heads, out)
    return out


def branch_split_hybrid_fwd(layout: Layout, shard: Shard, rank: int, plan: Plan, group=None,
                            rms_weight=None, rms_eps: float = 1e-6,
                            softmax: Callable = _default_softmax,
                            linear: Callable = _default_linear,
                            combine: Callable = _default_combine) -> torch.Tensor:
    """The branch-specialised split over the ranks of `group` (plan from
    branch_split_plan): returns this rank's token shard of the hybrid output,
    [B, |tokens[rank]|, H, d]."""
    B, H, d, L = layout.B, layout.H, layout.d, layout.L
    dev, dt, bt = shard.q.device, shard.q.dtype, shard.beta.dtype
    W = plan.world
    sh, lh = plan.soft_heads[rank], plan.lin_heads[rank]
    # uneven all-to-all: q, k, v to the softmax rank of each head; q, k, v,
    # beta to its linear rank (a rank is one or the other)
    send = []
    for p in range(W):
        if len(plan.soft_heads[p]):
            send.append([_heads(t, plan.soft_heads[p]) for t in (shard.q, shard.k, shard.v)])
        else:
            send.append([_heads(t, plan.lin_heads[p]) for t in (shard.q, shard.k, shard.v, shard.beta)])
    specs = []
    for p in range(W):
        n = len(plan.tokens[p])
        if len(sh):
            specs.append([((B, n, len(sh), d), dt)] * 3)
        else:
            specs.append([((B, n, len(lh), d), dt)] * 3 + [((B, n, len(lh)), bt)])
    got = exchange(send, specs, dev, group)
    if len(sh):
        q, k, v = [_assemble([g[i] for g in got], plan, B, L, len(sh), (d,), dt, dev) for i in range(3)]
        o_h = softmax(_layout_heads(layout, len(sh)), q, k, v, _text(shard.k_text, sh),
                      _text(shard.v_text, sh))
    else:
        q, k, v = [_assemble([g[i] for g in got], plan, B, L, len(lh), (d,), dt, dev) for i in range(3)]
        beta = _assemble([g[3] for g in got], plan, B, L, len(lh), (), bt, dev)
        o_h = linear(_layout_heads(layout, len(lh)), q, k, v, _text(shard.k_text, lh),
                     _text(shard.v_text, lh), beta, _text(shard.beta_text, lh))
    # reverse uneven all-to-all: each token shard gets o_soft from every softmax
    # rank and o_lin from every linear rank, in the branches' float32 (a bf16
    # exchange would add two roundings to the output beyond the op's bound)
    ot = o_h.dtype
    back = [[o_h[:, plan.tokens[p].start:plan.tokens[p].stop].contiguous()] for p in range(W)]
    n_mine = len(plan.tokens[rank])
    specs = [[((B, n_mine, len(plan.soft_heads[p]) or len(plan.lin_heads[p]), d), ot)]
             for p in range(W)]
    got = exchange(back, specs, dev, group)
    o_soft = torch.empty((B, n_mine, H, d), dtype=ot, device=dev)
    o_lin = torch.empty((B, n_mine, H, d), dtype=ot, device=dev)
    _scatter_heads({p: got[p][0] for p in range(W) if len(plan.soft_heads[p])}, plan.soft_heads, o_soft)
    _scatter_heads({p: got[p][0] for p in range(W) if len(plan.lin_heads[p])}, plan.lin_heads, o_lin)
    return combine(o_soft, o_lin, shard.g_s, shard.g_l, rms_weight, rms_eps)


def shard_of(inputs: Dict[str, torch.Tensor], plan: Plan, rank: int) -> Shard:
    """Rank `rank`'s token shard of a full layer input (the dict make_inputs
    returns); the text tensors are replicated."""
    tr = plan.tokens[rank]

    def cut(t):
        return t[:, tr.start:tr.stop].contiguous()
    return Shard(q=cut(inputs["q"]), k=cut(inputs["k"]), v=cut(inputs["v"]), beta=cut(inputs["beta"]),
                 g_s=cut(inputs["g_s"]), g_l=cut(inputs["g_l"]), k_text=inputs.get("k_text"),
                 v_text=inputs.get("v_text"), beta_text=inputs.get("beta_text"))
