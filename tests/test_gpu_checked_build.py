"""The bound-checked build (libvdn_checked.so: the same sources compiled with
-DVDN_BOUND_CHECKS). Its kernels check their global row, slot and chunk indices
and the schedule's key rows before each access; a failed check skips the access
and records VDN_ERR_BOUNDS in the device status word (no trap). On the small
workloads and every edge layout of the parity tests, through all three entry
points, no check may fire and every result must equal the regular library's
bit for bit (the checks do not touch the arithmetic)."""

import os

import pytest
import torch

from linear_attention_video_block_b200 import build as B
from linear_attention_video_block_b200 import vdn
from linear_attention_video_block_b200.synth import WORKLOADS, make_inputs

from test_gpu_parity import EDGE

pytestmark = pytest.mark.gpu

LAYOUTS = [("tiny-f32", *WORKLOADS["tiny-f32"][:2]), ("small-bf16", *WORKLOADS["small-bf16"][:2])] + \
    [(n, l, dt) for n, l, dt in EDGE]


def _run_all(layout, d):
    args = (layout, d["q"], d["k"], d["v"], d["k_text"], d["v_text"])
    o_soft = vdn.window_softmax_fwd(*args)
    o_lin = vdn.vda_scan_fwd(*args, d["beta"], d["beta_text"])
    out = vdn.hybrid_attn_fwd(*args, d["beta"], d["beta_text"], d["g_s"], d["g_l"])
    torch.cuda.synchronize()
    return o_soft, o_lin, out


@pytest.fixture(scope="module")
def checked_library():
    if not os.path.exists(B.LIB_CHECKED):
        B.build(checked=True)
    return B.LIB_CHECKED


@pytest.mark.parametrize("name,layout,dtype", LAYOUTS, ids=[x[0] for x in LAYOUTS])
def test_checked_build_passes_every_check(checked_library, name, layout, dtype):
    d = {k: t.cuda() for k, t in make_inputs(layout, dtype, 31).items()}
    ref = _run_all(layout, d)
    assert vdn.device_status() == 0
    saved_lib, saved_path = vdn._lib, vdn._LIB_PATH
    try:
        vdn._lib, vdn._LIB_PATH = None, checked_library
        got = _run_all(layout, d)
        status = vdn.device_status()
    finally:
        vdn._lib, vdn._LIB_PATH = saved_lib, saved_path
    assert status == 0
    for g, r in zip(got, ref):
        assert torch.equal(g, r)
