"""The allocation-free linear-branch entry point (vdn_vda_scan_fwd_noalloc),
for callers that cannot allocate device memory where they run the op. It must
give the same results as vdn_vda_scan_fwd, call after call, from its static
scratch array. This file is collected last so that a run stopping at the first
failure has already run every other test."""

import ctypes

import pytest
import torch

from linear_attention_video_block_b200 import vdn
from linear_attention_video_block_b200.synth import Layout, WORKLOADS, make_inputs

from conftest import bf16_storage_ratio, rel_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny-f32", "small-bf16"])
def test_noalloc_matches_workspace_entry_on_two_calls(name):
    layout, dtype, seed = WORKLOADS[name]
    d = {k: t.to("cuda") for k, t in make_inputs(layout, dtype, seed).items()}
    args = (layout, d["q"], d["k"], d["v"], d["k_text"], d["v_text"], d["beta"], d["beta_text"])
    ref, ref_states = vdn.vda_scan_fwd(*args, want_states=True)
    ref = ref.double().cpu().numpy()
    ref_states = ref_states.double().cpu().numpy()
    J = -(-layout.F // layout.c)
    for call in range(2):
        o = torch.full_like(d["q"], float("nan"))
        st = torch.full((layout.B, layout.H, 2, J, layout.d, layout.d), float("nan"),
                        dtype=torch.float32, device="cuda")
        vdn.vda_scan_fwd_noalloc(*args, o_lin=o, chunk_states=st if call == 1 else None)
        torch.cuda.synchronize()
        got = o.double().cpu().numpy()
        if dtype == "f32":
            assert rel_err(got, ref) <= 1e-4, call
        else:
            assert bf16_storage_ratio(got, ref, allowance=2e-2) <= 1.0, call
        if call == 1:
            assert rel_err(st.double().cpu().numpy(), ref_states) <= 1e-4
    assert vdn.device_status() == 0


def test_noalloc_rejects_layouts_beyond_the_scratch():
    """480p-like needs 78 MiB of scratch, more than the 64 MiB array: refused,
    nothing launched."""
    layout, dtype, seed = WORKLOADS["480p-bf16"]
    small = Layout(B=layout.B, F=layout.F, N=8, T=layout.T, c=layout.c, H=layout.H, d=layout.d)
    d = {k: t.to("cuda") for k, t in make_inputs(small, dtype, seed).items()}
    o = torch.empty_like(d["q"])
    f = vdn.lib().vdn_vda_scan_fwd_noalloc
    f.argtypes = [ctypes.POINTER(vdn._CLayout), ctypes.c_int] + [ctypes.c_void_p] * 10
    f.restype = ctypes.c_int
    code = f(ctypes.byref(vdn._clayout(small)), 1, *[ctypes.c_void_p(d[k].data_ptr()) for k in
             ("q", "k", "v", "k_text", "v_text", "beta", "beta_text")],
             ctypes.c_void_p(o.data_ptr()), None, None)
    assert code == 3  # VDN_ERR_WORKSPACE
