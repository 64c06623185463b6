"""The failure path of the bounded waits, exercised without a fault.

Every wait between the roles of the tensor-core kernels (TMA producer, MMA
issuer, softmax / scaler / drain warps) is bounded; when it gives up, the
kernel records VDN_ERR_TIMEOUT in the status word, its roles leave their loops,
it waits for its own copies and MMAs (those waits keep the 4 s limit) and frees
TMEM before it exits. Here the role-wait limit is set to one nanosecond, so the
first wait that does not succeed at once gives up; the test checks that the
status word reports the timeout, that nothing faults, and that after restoring
the limit the same call reproduces its earlier result bit for bit (TMEM and the
barriers were left clean)."""

import pytest
import torch

from linear_attention_video_block_b200 import vdn
from linear_attention_video_block_b200.synth import Layout, make_inputs

pytestmark = pytest.mark.gpu

VDN_ERR_TIMEOUT = 5

CASES = [
    # (name, layout): the window kernel (d = 64 and d = 128), the tensor-core
    # Gram and readout (linear branch, d = 128)
    ("window-d64", Layout(B=1, F=9, N=300, T=40, c=3, H=2, d=64)),
    ("window-d128", Layout(B=1, F=9, N=300, T=40, c=3, H=2, d=128)),
    ("linear-d128", Layout(B=1, F=9, N=300, T=40, c=3, H=2, d=128)),
]


def _call(name, layout, d):
    if name.startswith("window"):
        return vdn.window_softmax_fwd(layout, d["q"], d["k"], d["v"], d["k_text"], d["v_text"])
    return vdn.vda_scan_fwd(layout, d["q"], d["k"], d["v"], d["k_text"], d["v_text"], d["beta"],
                            d["beta_text"])


@pytest.mark.parametrize("name,layout", CASES, ids=[c[0] for c in CASES])
def test_role_wait_timeout_reports_and_recovers(name, layout):
    d = {k: t.cuda() for k, t in make_inputs(layout, "bf16", 21).items()}
    assert vdn.device_status() == 0
    ref = _call(name, layout, d).clone()
    torch.cuda.synchronize()
    assert vdn.device_status() == 0
    try:
        vdn.set_wait_limit_ns(1)
        _call(name, layout, d)
        torch.cuda.synchronize()
        status = vdn.device_status()
    finally:
        vdn.set_wait_limit_ns(0)
    assert status == VDN_ERR_TIMEOUT
    again = _call(name, layout, d)
    torch.cuda.synchronize()
    assert vdn.device_status() == 0
    assert torch.equal(again, ref)
