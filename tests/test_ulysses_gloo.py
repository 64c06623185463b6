"""Sequence-parallel routing of the hybrid layer (linear_attention_video_block_b200
.ulysses) on CPU processes with the gloo backend.

The routing only moves data; the per-head computation is the library's entry
points on GPUs. Here the float64 oracle stands in for those entry points
(injected by the test), so that what is checked is the routing itself: the
token shards and head shards, the uneven all-to-all of the branch-specialised
split (project page, "Parallelization & Few-Step Generation": softmax GPUs and
linear-branch GPUs, then a reverse all-to-all to the token shards), and the
reassembly. Every rank's token shard of the routed output must equal the same
rows of the single-process oracle output.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from linear_attention_video_block_b200 import ulysses as U
from linear_attention_video_block_b200.synth import Layout, make_inputs
from oracle import vdn_oracle as O


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _np(t):
    return None if t is None else t.detach().double().numpy()


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a))


# the oracle in the shape of the library's entry points (test side only)
def oracle_hybrid(lay, q, k, v, kt, vt, beta, bt, gs, gl, w, eps):
    r = O.hybrid(_np(q), _np(k), _np(v), _np(kt), _np(vt), _np(beta), _np(bt), _np(gs), _np(gl),
                 lay.F, lay.N, lay.c, eps=eps, weight=_np(w))
    return _t(r["out"])


def oracle_softmax(lay, q, k, v, kt, vt):
    return _t(O.softmax_branch(_np(q), _np(k), _np(v), _np(kt), _np(vt), lay.F, lay.N, lay.c))


def oracle_linear(lay, q, k, v, kt, vt, beta, bt):
    return _t(O.linear_branch(_np(q), _np(k), _np(v), _np(kt), _np(vt), _np(beta), _np(bt),
                              lay.F, lay.N, lay.c))


def oracle_combine(o_soft, o_lin, gs, gl, w, eps):
    return _t(O.combine(_np(o_soft), _np(o_lin), _np(gs), _np(gl), eps=eps, weight=_np(w))[0])


def _inputs(lay, seed):
    inp = make_inputs(lay, "f32", seed)
    # float64 end to end: the routing must not change a single bit
    return {k: (v.double() if v.dtype == torch.float32 else v) for k, v in inp.items()}


def _worker(rank, world, port, lay, seed, mode, n_soft, weighted):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = _inputs(lay, seed)
        w = torch.linspace(0.5, 1.5, lay.d, dtype=torch.float64) if weighted else None
        eps = 1e-5 if weighted else 1e-6
        if mode == "ulysses":
            plan = U.ulysses_plan(lay, world)
            shard = U.shard_of(inp, plan, rank)
            out = U.ulysses_hybrid_fwd(lay, shard, rank, plan, rms_weight=w, rms_eps=eps,
                                       hybrid=oracle_hybrid)
        else:
            plan = U.branch_split_plan(lay, world, n_soft)
            shard = U.shard_of(inp, plan, rank)
            out = U.branch_split_hybrid_fwd(lay, shard, rank, plan, rms_weight=w, rms_eps=eps,
                                            softmax=oracle_softmax, linear=oracle_linear,
                                            combine=oracle_combine)
        ref = O.hybrid(*[_np(inp[k]) for k in ("q", "k", "v", "k_text", "v_text", "beta",
                                                "beta_text", "g_s", "g_l")],
                       lay.F, lay.N, lay.c, eps=eps, weight=_np(w))["out"]
        tr = plan.tokens[rank]
        assert tuple(out.shape) == (lay.B, len(tr), lay.H, lay.d)
        np.testing.assert_allclose(out.numpy(), ref[:, tr.start:tr.stop], rtol=0, atol=1e-12)
    finally:
        dist.destroy_process_group()


CASES = [
    # (mode, world, n_soft, layout, weighted)
    ("ulysses", 2, 0, Layout(B=1, F=8, N=6, T=3, c=2, H=4, d=16), False),
    ("ulysses", 2, 0, Layout(B=2, F=7, N=5, T=0, c=3, H=3, d=16), True),   # ragged heads/tokens, no text
    ("branch", 3, 2, Layout(B=1, F=8, N=6, T=3, c=2, H=4, d=16), False),   # 2 softmax + 1 linear
    ("branch", 3, 1, Layout(B=2, F=9, N=5, T=4, c=2, H=5, d=16), True),    # 1 softmax + 2 linear, ragged
]


@pytest.mark.parametrize("mode,world,n_soft,lay,weighted", CASES,
                         ids=[f"{c[0]}-w{c[1]}-s{c[2]}-H{c[3].H}" for c in CASES])
def test_routed_layer_equals_single_process(mode, world, n_soft, lay, weighted):
    mp.spawn(_worker, args=(world, _free_port(), lay, 11, mode, n_soft, weighted), nprocs=world,
             join=True)


def test_plans_cover_every_token_and_head_once():
    lay = Layout(B=1, F=36, N=4032, T=512, c=5, H=40, d=128)
    for world in (1, 2, 3, 8):
        p = U.ulysses_plan(lay, world)
        assert sorted(t for r in p.tokens for t in r) == list(range(lay.L))
        assert sorted(h for r in p.soft_heads for h in r) == list(range(lay.H))
        assert p.soft_heads == p.lin_heads
    for world, n_soft in ((8, 5), (8, 7), (3, 2), (2, 1)):
        p = U.branch_split_plan(lay, world, n_soft)
        assert sorted(t for r in p.tokens for t in r) == list(range(lay.L))
        assert sorted(h for r in p.soft_heads for h in r) == list(range(lay.H))
        assert sorted(h for r in p.lin_heads for h in r) == list(range(lay.H))
        for r in range(world):  # a rank works on one branch only
            assert (len(p.soft_heads[r]) > 0) != (len(p.lin_heads[r]) > 0)
    with pytest.raises(ValueError):
        U.branch_split_plan(lay, 4, 4)
    with pytest.raises(ValueError):
        U.ulysses_plan(Layout(B=1, F=3, N=2, T=0, c=1, H=2, d=16), 3)


def test_routing_defaults_are_the_library_entry_points():
    """Without injected functions the routings call the CUDA entry points of
    the binding (there is no CPU path): on a host without a GPU they fail at
    the device check."""
    lay = Layout(B=1, F=4, N=4, T=2, c=2, H=2, d=64)
    inp = make_inputs(lay, "bf16", 3)
    plan = U.ulysses_plan(lay, 1)
    shard = U.shard_of(inp, plan, 0)
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    with pytest.raises(RuntimeError, match="CUDA device"):
        U.ulysses_hybrid_fwd(lay, shard, 0, plan)
    with pytest.raises(RuntimeError, match="CUDA device"):
        U.branch_split_hybrid_fwd(lay, shard, 0, U.Plan(1, plan.tokens, plan.soft_heads,
                                                         [range(0, 0)]))
