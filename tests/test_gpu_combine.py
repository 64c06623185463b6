"""GPU parity of the gated combine entry (vdn_gated_combine_fwd) and of the
pieces a branch-specialised sequence-parallel split runs: the softmax entry on
some heads, the linear entry on others, and the combine on token shards.

Bounds as in test_gpu_parity: fp32 max|err|/RMS <= 1e-4; bf16 `out` raw
max|err|/RMS <= 2e-2 (check_out_bf16)."""

import numpy as np
import pytest
import torch

from linear_attention_video_block_b200 import ulysses as U
from linear_attention_video_block_b200 import vdn
from linear_attention_video_block_b200.synth import Layout, WORKLOADS, make_inputs
from oracle import vdn_oracle as O

from conftest import check_out_bf16, rel_err

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().cpu().double().numpy()


@pytest.mark.parametrize("dtype,d,weighted", [("f32", 16, False), ("f32", 128, True),
                                              ("bf16", 64, True), ("bf16", 128, False)])
def test_gated_combine_matches_oracle(dtype, d, weighted):
    """out = sigmoid(g_s) o_soft + sigmoid(g_l) RMSNorm(o_lin) on random branch
    outputs, including all-zero o_lin rows (boundary frames) and a ragged row
    count."""
    g = torch.Generator().manual_seed(d)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    shape = (2, 333, 3, d)
    t = {k: torch.randn(shape, generator=g).to(tdt if k.startswith("g") else torch.float32)
         for k in ("o_soft", "o_lin", "g_s", "g_l")}
    t["o_lin"][:, :17] = 0
    w = torch.linspace(0.5, 1.5, d) if weighted else None
    eps = 1e-5 if weighted else 1e-6
    dev = {k: v.cuda() for k, v in t.items()}
    out = vdn.gated_combine_fwd(dev["o_soft"], dev["o_lin"], dev["g_s"], dev["g_l"],
                                rms_weight=None if w is None else w.cuda(), rms_eps=eps)
    torch.cuda.synchronize()
    ref = O.combine(_np(t["o_soft"]), _np(t["o_lin"]), _np(t["g_s"]), _np(t["g_l"]), eps=eps,
                    weight=None if w is None else w.double().numpy())[0]
    if dtype == "f32":
        assert rel_err(_np(out), ref) <= 1e-4
    else:
        check_out_bf16(_np(out), ref, {})
    assert vdn.device_status() == 0


def test_gated_combine_of_the_branch_entries_equals_the_hybrid_entry():
    """The two branch entries followed by the combine on three token shards (what
    the ranks of a branch-specialised split run) give the hybrid output within
    the bf16 bound against the oracle."""
    layout, dtype, seed = WORKLOADS["small-bf16"]
    inp = make_inputs(layout, dtype, seed)
    d = {k: v.cuda() for k, v in inp.items()}
    o_soft = vdn.window_softmax_fwd(layout, d["q"], d["k"], d["v"], d["k_text"], d["v_text"],
                                    out_f32=True)
    o_lin = vdn.vda_scan_fwd(layout, d["q"], d["k"], d["v"], d["k_text"], d["v_text"], d["beta"],
                             d["beta_text"], out_f32=True)
    assert o_soft.dtype == torch.float32 and o_lin.dtype == torch.float32
    # the float32 forms agree with the io-dtype entries up to their rounding
    o_soft_b = vdn.window_softmax_fwd(layout, d["q"], d["k"], d["v"], d["k_text"], d["v_text"])
    o_lin_b = vdn.vda_scan_fwd(layout, d["q"], d["k"], d["v"], d["k_text"], d["v_text"], d["beta"],
                               d["beta_text"])
    assert torch.equal(o_soft.to(torch.bfloat16), o_soft_b)
    assert torch.equal(o_lin.to(torch.bfloat16), o_lin_b)
    out = torch.empty_like(d["q"])
    for tr in U.even_ranges(layout.L, 3):  # three token shards
        sl = slice(tr.start, tr.stop)
        out[:, sl] = vdn.gated_combine_fwd(o_soft[:, sl].contiguous(), o_lin[:, sl].contiguous(),
                                           d["g_s"][:, sl].contiguous(), d["g_l"][:, sl].contiguous())
    torch.cuda.synchronize()
    a = {k: _np(v) for k, v in inp.items()}
    ref = O.hybrid(a["q"], a["k"], a["v"], a["k_text"], a["v_text"], a["beta"], a["beta_text"],
                   a["g_s"], a["g_l"], layout.F, layout.N, layout.c)["out"]
    res = {}
    check_out_bf16(_np(out), ref, res)
    assert res["out_rule"] == "raw"
    assert vdn.device_status() == 0


def test_ulysses_single_rank_is_the_hybrid_entry():
    """With one rank the Ulysses routing is the identity around
    vdn_hybrid_attn_fwd: same output bit for bit."""
    layout, dtype, seed = WORKLOADS["small-bf16"]
    d = {k: v.cuda() for k, v in make_inputs(layout, dtype, seed).items()}
    plan = U.ulysses_plan(layout, 1)
    out = U.ulysses_hybrid_fwd(layout, U.shard_of(d, plan, 0), 0, plan)
    ref = vdn.hybrid_attn_fwd(layout, d["q"], d["k"], d["v"], d["k_text"], d["v_text"], d["beta"],
                              d["beta_text"], d["g_s"], d["g_l"])
    assert torch.equal(out, ref)
