"""GPU parity of the joint text-video-audio layer (vdn_joint_softmax_fwd,
vdn_joint_attn_fwd) against the float64 oracle on the same seeded inputs.

Video rows: the softmax branch also sees every audio key; the linear branch is
unchanged (audio is never written into the VDA states). Text and audio query
rows: the dense softmax over every video, text and audio key. Bounds as in
test_gpu_parity: fp32 max|err|/RMS <= 1e-4; the bf16 output `out` to a raw
max|err|/RMS(out) <= 2e-2 wherever rounding the exact result to bf16 stays
within 2e-2 (the 480p-like and 768p-like layers assert that this raw rule
applied), the other bf16 results to 2e-2 RMS beyond their own storage
rounding; lse <= 1e-3 absolute (1e-4 for fp32).
"""

import numpy as np
import pytest
import torch

from linear_attention_video_block_b200 import vdn
from linear_attention_video_block_b200.synth import (Layout, WORKLOADS, audio_tokens, make_context,
                                                     make_decay, make_inputs)
from oracle import vdn_oracle as O

from conftest import bf16_storage_ratio, check_out_bf16, rel_err

pytestmark = pytest.mark.gpu


def _np(t, heads=None):
    if t is None:
        return None
    t = t.detach().to("cpu")
    if heads is not None:
        t = t[:, :, heads]
    return t.to(torch.float64).numpy()


def _sample_rows(layout, per_frame, seed=0):
    rng = np.random.default_rng(seed)
    F, N = layout.F, layout.N
    rows = set()
    for f in range(F):
        base = f * N
        rows |= {base, base + N - 1}
        rows |= set((base + rng.integers(0, N, size=per_frame)).tolist())
    return np.array(sorted(rows))


def _check_joint(layout, dtype, inp, cx, heads=None, rows=None, alpha=None, text_rows=True,
                 audio_rows=True):
    d = {k: v.to("cuda") for k, v in inp.items()}
    c = {k: v.to("cuda") for k, v in cx.items()}
    ka = c["k_audio"] if c["k_audio"].shape[1] else None
    va = c["v_audio"] if ka is not None else None
    qt = c["q_text"] if (text_rows and layout.T > 0) else None
    qa = c["q_audio"] if (audio_rows and ka is not None) else None
    sm = vdn.joint_softmax_fwd(layout, d["q"], d["k"], d["v"], d["k_text"], d["v_text"],
                               k_audio=ka, v_audio=va, q_text=qt, q_audio=qa, want_lse=True)
    out_soft = torch.empty_like(d["q"])
    out_lin = torch.empty_like(d["q"])
    alpha_d = None if alpha is None else alpha.to("cuda")
    out, o_text, o_audio = vdn.joint_attn_fwd(
        layout, d["q"], d["k"], d["v"], d["k_text"], d["v_text"], d["beta"], d["beta_text"],
        d["g_s"], d["g_l"], k_audio=ka, v_audio=va, q_text=qt, q_audio=qa, alpha=alpha_d,
        out_soft=out_soft, out_lin=out_lin)
    torch.cuda.synchronize()
    assert vdn.device_status() == 0
    hsel = list(range(layout.H)) if heads is None else heads
    a = {k: _np(v, hsel) for k, v in inp.items()}
    x = {k: _np(v, hsel) for k, v in cx.items()}
    F, N, c_ = layout.F, layout.N, layout.c
    kx = x["k_audio"] if ka is not None else None
    vx = x["v_audio"] if ka is not None else None
    ref_soft, ref_lse = O.softmax_branch(a["q"], a["k"], a["v"], a["k_text"], a["v_text"], F, N, c_,
                                         rows=rows, return_lse=True, k_audio=kx, v_audio=vx)
    ref_lin = O.linear_branch(a["q"], a["k"], a["v"], a["k_text"], a["v_text"], a["beta"],
                              a["beta_text"], F, N, c_, alpha=_np(alpha, hsel))
    ref_out, ref_gs, ref_gl = O.combine(ref_soft, ref_lin, a["g_s"], a["g_l"])
    comp = {"out": (out, ref_out, None), "o_soft": (sm["o_soft"], ref_soft, None),
            "out_soft": (out_soft, ref_gs, "out"), "out_lin": (out_lin, ref_gl, "out")}
    lses = {"lse": (sm["lse"], ref_lse)}
    for name, qrows, got_sm, got_j, lse in (("o_text", qt, sm["o_text"], o_text, sm["lse_text"]),
                                           ("o_audio", qa, sm["o_audio"], o_audio, sm["lse_audio"])):
        if qrows is None:
            assert got_j is None
            continue
        ref, rl = O.context_rows(x["q_text" if name == "o_text" else "q_audio"], a["k"], a["v"],
                                 a["k_text"], a["v_text"], kx, vx, return_lse=True)
        comp[name] = (got_sm, ref, None)
        comp[name + "_joint"] = (got_j, ref, None)
        lses[name.replace("o_", "lse_")] = (lse, rl)
    rms_out = float(np.sqrt(np.nanmean(ref_out ** 2)))
    res = {}
    if dtype == "bf16":
        # the op's output: raw max|err|/RMS <= 2e-2 (see check_out_bf16)
        check_out_bf16(_np(out, hsel), ref_out, res)
    for key, (g, r, scale_of) in comp.items():
        gv = _np(g, hsel)
        res[key] = rel_err(gv, r)
        if dtype == "bf16" and key != "out":
            res[key + "_storage_ratio"] = bf16_storage_ratio(
                gv, r, allowance=2e-2, rms=rms_out if scale_of == "out" else None)
    for key, (g, r) in lses.items():
        res[key] = float(np.nanmax(np.abs(g.cpu().double().numpy()[:, :, hsel] - r)))
    print(layout, dtype, {k: (round(v, 6) if isinstance(v, float) else v) for k, v in res.items()})
    for key in comp:
        if dtype == "f32":
            assert res[key] <= 1e-4, (key, res)
        elif key != "out":
            assert res[key + "_storage_ratio"] <= 1.0, (key, res)
    for key in lses:
        assert res[key] <= (1e-4 if dtype == "f32" else 1e-3), (key, res)
    return res


@pytest.mark.parametrize("name,A", [("tiny-f32", 3), ("small-bf16", 13), ("small-bf16", 130)])
def test_joint_small_full(name, A):
    layout, dtype, seed = WORKLOADS[name]
    _check_joint(layout, dtype, make_inputs(layout, dtype, seed), make_context(layout, A, dtype, seed + 7))


JOINT_EDGE = [
    # (name, layout, dtype, A, text_rows, audio_rows)
    ("no-text-audio-only", Layout(B=1, F=9, N=70, T=0, c=2, H=2, d=128), "bf16", 40, True, True),
    ("text-rows-only", Layout(B=2, F=7, N=200, T=130, c=1, H=2, d=128), "bf16", 5, True, False),
    ("audio-rows-only", Layout(B=1, F=3, N=50, T=7, c=1, H=2, d=64), "bf16", 257, False, True),
    ("one-audio-one-frame", Layout(B=1, F=1, N=37, T=5, c=2, H=2, d=64), "bf16", 1, True, True),
    ("one-token-frames", Layout(B=1, F=12, N=1, T=2, c=2, H=3, d=64), "bf16", 2, True, True),
    ("no-audio", Layout(B=1, F=6, N=40, T=9, c=8, H=1, d=128), "bf16", 0, True, False),
    ("f32-d32", Layout(B=1, F=10, N=33, T=6, c=3, H=2, d=32), "f32", 4, True, True),
    ("f32-d16-no-text", Layout(B=2, F=13, N=8, T=0, c=4, H=2, d=16), "f32", 9, False, True),
]


@pytest.mark.parametrize("name,layout,dtype,A,tr,ar", JOINT_EDGE, ids=[e[0] for e in JOINT_EDGE])
def test_joint_edge_layouts(name, layout, dtype, A, tr, ar):
    seed = 300 + len(name)
    _check_joint(layout, dtype, make_inputs(layout, dtype, seed), make_context(layout, A, dtype, seed + 1),
                 text_rows=tr, audio_rows=ar)


def test_joint_with_decay():
    layout, dtype, seed = WORKLOADS["small-bf16"]
    _check_joint(layout, dtype, make_inputs(layout, dtype, seed), make_context(layout, 21, dtype, seed + 7),
                 alpha=make_decay(layout, seed + 1))


@pytest.mark.parametrize("name", ["480p-bf16", "768p-bf16"])
def test_joint_full_size_sampled(name):
    """The 480p-like and 768p-like layers with their audio length (118 and 203
    tokens) and every text and audio query row; sampled video rows of heads
    {0, H-1}."""
    layout, dtype, seed = WORKLOADS[name]
    A = audio_tokens(layout.F)
    res = _check_joint(layout, dtype, make_inputs(layout, dtype, seed),
                       make_context(layout, A, dtype, seed + 7), heads=[0, layout.H - 1],
                       rows=_sample_rows(layout, 12))
    assert res["out_rule"] == "raw"


def test_joint_without_context_is_the_plain_hybrid():
    """A = 0 and no context rows: the joint entry reproduces vdn_hybrid_attn_fwd
    bit for bit (same kernels, the context groups are empty)."""
    layout, dtype, seed = WORKLOADS["small-bf16"]
    d = {k: v.to("cuda") for k, v in make_inputs(layout, dtype, seed).items()}
    args = (layout, d["q"], d["k"], d["v"], d["k_text"], d["v_text"], d["beta"], d["beta_text"],
            d["g_s"], d["g_l"])
    a = vdn.hybrid_attn_fwd(*args)
    b, t, au = vdn.joint_attn_fwd(*args)
    assert t is None and au is None
    assert torch.equal(a, b)
    s1 = vdn.window_softmax_fwd(layout, d["q"], d["k"], d["v"], d["k_text"], d["v_text"])
    s2 = vdn.joint_softmax_fwd(layout, d["q"], d["k"], d["v"], d["k_text"], d["v_text"])["o_soft"]
    assert torch.equal(s1, s2)
