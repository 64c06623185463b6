"""GPU parity of the FP8 (e4m3) softmax branch (vdn_window_softmax_fwd_fp8)
against the float64 oracle.

The inputs are drawn with the usual recipe, then stored as e4m3 with one scale
per tensor (text shares the scales of k and v); the oracle receives exactly the
dequantized values, so input quantization is not counted as error. What the
kernel adds is the e4m3 rounding of the softmax weights P (3 mantissa bits:
relative error up to 2^-4 per weight; the float32 row sum is taken before
rounding) and the bf16 output. That rounding does not average out relative to
the output: over N similar weights both the output and the error shrink like
1/sqrt(N), so the relative error stays at the weights' own level (emulating
e4m3 weights in float64 on these inputs gives 2.5 % RMS, 10.6 % max/RMS).
Bounds derived from that arithmetic:
  - per element, the worst case: |gpu - oracle| <= 2^-8 |oracle| (bf16 output)
    + 2^-4 sum_j p_j |v_j| (every weight off by its largest rounding);
  - RMS(gpu - oracle) / RMS(oracle) <= 4e-2 (2.6 % expected from uniform
    rounding within e4m3 binades, plus margin), which catches layout errors
    (a wrong operand layout gives errors of the order of the output itself);
  - LSE (from the float32 weights) within 1e-3.
"""

import numpy as np
import pytest
import torch

from linear_attention_video_block_b200 import vdn
from linear_attention_video_block_b200.synth import Layout, WORKLOADS, make_inputs, quantize_e4m3
from oracle import vdn_oracle as O

from conftest import rel_err

pytestmark = pytest.mark.gpu


def _run(layout, seed, heads=None, rows=None):
    inp = make_inputs(layout, "bf16", seed)
    (q8,), sq = quantize_e4m3(inp["q"])
    (k8, kt8), sk = quantize_e4m3(inp["k"], inp["k_text"])
    (v8, vt8), sv = quantize_e4m3(inp["v"], inp["v_text"])
    d = [t.to("cuda") for t in (q8, k8, v8, kt8, vt8)]
    o, lse = vdn.window_softmax_fwd_fp8(layout, *d, sq, sk, sv, want_lse=True)
    torch.cuda.synchronize()
    assert vdn.device_status() == 0
    hsel = list(range(layout.H)) if heads is None else heads
    deq = lambda t8, s: (t8.float() * s).double()[:, :, hsel].numpy()
    qd, kd, vd, ktd, vtd = deq(q8, sq), deq(k8, sk), deq(v8, sv), deq(kt8, sk), deq(vt8, sv)
    F, N, c = layout.F, layout.N, layout.c
    ref, ref_lse = O.softmax_branch(qd, kd, vd, ktd, vtd, F, N, c, rows=rows, return_lse=True)
    ref_abs = O.softmax_branch(qd, kd, np.abs(vd), ktd, np.abs(vtd), F, N, c, rows=rows)
    got = o.cpu().double()[:, :, hsel].numpy()
    m = ~np.isnan(ref)
    err = np.abs(got[m] - ref[m])
    res = {"o_soft": rel_err(got, ref),
           "rms_rel": float(np.sqrt(np.mean(err ** 2)) / np.sqrt(np.mean(ref[m] ** 2))),
           "bound_ratio": float(np.max(err / (2.0 ** -8 * np.abs(ref[m]) + 2.0 ** -4 * ref_abs[m]))),
           "lse": float(np.nanmax(np.abs(lse.cpu().double().numpy()[:, :, hsel] - ref_lse)))}
    print(layout, {k: round(v, 6) for k, v in res.items()})
    assert res["bound_ratio"] <= 1.0, res
    assert res["rms_rel"] <= 4e-2, res
    assert res["lse"] <= 1e-3, res
    return res


FP8_CASES = [
    ("small-d128", Layout(B=1, F=20, N=256, T=64, c=5, H=4, d=128)),
    ("no-text", Layout(B=1, F=9, N=70, T=0, c=2, H=2, d=128)),
    ("one-frame", Layout(B=1, F=1, N=37, T=5, c=2, H=2, d=128)),
    ("three-frames-c1", Layout(B=2, F=3, N=130, T=7, c=1, H=1, d=128)),
    ("ragged-c1", Layout(B=1, F=7, N=200, T=130, c=1, H=2, d=128)),
]


@pytest.mark.parametrize("name,layout", FP8_CASES, ids=[c[0] for c in FP8_CASES])
def test_fp8_window_small(name, layout):
    _run(layout, seed=400 + len(name))


@pytest.mark.parametrize("name", ["480p-bf16", "768p-bf16"])
def test_fp8_window_full_size_sampled(name):
    layout, _, seed = WORKLOADS[name]
    rng = np.random.default_rng(0)
    rows = set()
    for f in range(layout.F):
        base = f * layout.N
        rows |= {base, base + layout.N - 1}
        rows |= set((base + rng.integers(0, layout.N, size=8)).tolist())
    _run(layout, seed, heads=[0, layout.H - 1], rows=np.array(sorted(rows)))
