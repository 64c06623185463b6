"""The allocation-free linear-branch entry point (vdn_vda_scan_fwd_noalloc),
for callers that cannot allocate device memory where they run the op (a
plugin whose host engine owns all device memory, a serving loop that allows
no allocation after start-up). It launches the same kernels as
vdn_vda_scan_fwd on the same inputs, only with its scratch in a static device
array, so its results must equal that entry's bit for bit, call after call,
whatever the previous call left in the array. This file is collected last so
that a run stopping at the first failure has already run every other test."""

import pytest
import torch

from linear_attention_video_block_b200 import vdn
from linear_attention_video_block_b200.synth import Layout, WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny-f32", "small-bf16"])
def test_noalloc_matches_workspace_entry_on_two_calls(name):
    layout, dtype, seed = WORKLOADS[name]
    d = {k: t.to("cuda") for k, t in make_inputs(layout, dtype, seed).items()}
    args = (layout, d["q"], d["k"], d["v"], d["k_text"], d["v_text"], d["beta"], d["beta_text"])
    ref, ref_states = vdn.vda_scan_fwd(*args, want_states=True)
    J = -(-layout.F // layout.c)
    for call in range(2):
        o = torch.full_like(d["q"], float("nan"))
        st = torch.full((layout.B, layout.H, 2, J, layout.d, layout.d), float("nan"),
                        dtype=torch.float32, device="cuda")
        # the first call keeps the chunk states in the static array, the
        # second writes them to the caller's tensor
        vdn.vda_scan_fwd_noalloc(*args, o_lin=o, chunk_states=st if call == 1 else None)
        torch.cuda.synchronize()
        assert torch.equal(o, ref), call
        if call == 1:
            assert torch.equal(st, ref_states)
    assert vdn.device_status() == 0


def test_noalloc_rejects_layouts_beyond_the_scratch():
    """480p-like needs 78 MiB of scratch, more than the 64 MiB array: refused
    with VDN_ERR_WORKSPACE, nothing launched."""
    layout, dtype, seed = WORKLOADS["480p-bf16"]
    small = Layout(B=layout.B, F=layout.F, N=8, T=layout.T, c=layout.c, H=layout.H, d=layout.d)
    d = {k: t.to("cuda") for k, t in make_inputs(small, dtype, seed).items()}
    o = torch.empty_like(d["q"])
    with pytest.raises(vdn.VdnError) as e:
        vdn.vda_scan_fwd_noalloc(small, d["q"], d["k"], d["v"], d["k_text"], d["v_text"], d["beta"],
                                 d["beta_text"], o)
    assert e.value.code == 3  # VDN_ERR_WORKSPACE
