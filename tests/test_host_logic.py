"""Host-side logic of the CUDA path, checked on the CPU (no GPU calls):
the exported C ABI, its argument validation, and the query-group schedule the
kernels use, against the oracle's key sets and read states."""

import ctypes
import os
import re
import subprocess
import tempfile

import pytest

from oracle import vdn_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vdn.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(vdn_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from linear_attention_video_block_b200 import vdn
    return vdn.lib()


def test_library_exports_every_declared_function(lib):
    names = _declared_functions()
    assert {"vdn_window_softmax_fwd", "vdn_vda_scan_fwd", "vdn_hybrid_attn_fwd"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code in range(7):
        assert lib.vdn_status_string(code)
    assert lib.vdn_status_string(99) == b"unknown status"
    assert lib.vdn_last_cuda_error() == b"no CUDA error"


def _layout(**kw):
    from linear_attention_video_block_b200 import vdn
    base = dict(B=1, F=8, N=16, T=4, c=2, H=1, d=16)
    base.update(kw)
    return vdn._CLayout(*[base[k] for k in ("B", "F", "N", "T", "c", "H", "d")])


FAKE = ctypes.c_void_p(1 << 20)        # never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p((1 << 20) + 8)


def test_validation_rejects_before_any_launch(lib):
    """Every rejected call returns before touching CUDA (these run without a GPU)."""
    w = lib.vdn_window_softmax_fwd
    ok = _layout()
    args = [FAKE] * 6 + [None, None]
    assert w(ctypes.byref(_layout(B=0)), 0, *args) == 1          # invalid layout
    assert w(ctypes.byref(_layout(c=0)), 0, *args) == 1
    assert w(None, 0, *args) == 1
    assert w(ctypes.byref(ok), 7, *args) == 2                    # unknown dtype
    assert w(ctypes.byref(_layout(d=16)), 1, *args) == 2         # bf16 needs d in {64,128}
    assert w(ctypes.byref(_layout(d=48)), 0, *args) == 2
    assert w(ctypes.byref(ok), 0, None, FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == 1
    assert w(ctypes.byref(ok), 0, FAKE, FAKE, FAKE, None, FAKE, FAKE, None, None) == 1  # T>0 needs text
    assert w(ctypes.byref(ok), 0, MISALIGNED, FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == 2
    need = lib.vdn_workspace_bytes(ctypes.byref(ok), 0)
    assert need > 0 and lib.vdn_workspace_bytes(ctypes.byref(_layout(N=0)), 0) == 0
    v = lib.vdn_vda_scan_fwd
    vargs = [FAKE] * 8 + [None, FAKE]
    assert v(ctypes.byref(ok), 0, *vargs, 256, None) == 3        # short workspace
    assert v(ctypes.byref(ok), 0, *vargs[:-1], None, need, None) == 3
    h = lib.vdn_hybrid_attn_fwd
    hargs = [FAKE] * 9 + [None, ctypes.c_float(1e-6), FAKE, None, None, FAKE]
    assert h(ctypes.byref(ok), 0, *hargs, need - 1, None) == 3
    assert h(ctypes.byref(ok), 0, *hargs[:9], None, ctypes.c_float(-1.0), FAKE, None, None, FAKE, need, None) == 1


def test_decay_entries_validate_alpha(lib):
    """The _decay entry points require alpha and its alignment; everything else is
    validated as in the plain entries (no GPU is touched by any of these)."""
    ok = _layout()
    need = lib.vdn_workspace_bytes(ctypes.byref(ok), 0)
    v = lib.vdn_vda_scan_fwd_decay
    pre = [FAKE] * 7                                    # q k v kt vt beta beta_text
    assert v(ctypes.byref(ok), 0, *pre, None, FAKE, None, FAKE, need, None) == 1
    assert v(ctypes.byref(ok), 0, *pre, MISALIGNED, FAKE, None, FAKE, need, None) == 2
    assert v(ctypes.byref(ok), 0, *pre, FAKE, FAKE, None, FAKE, 256, None) == 3
    assert v(ctypes.byref(_layout(F=0)), 0, *pre, FAKE, FAKE, None, FAKE, need, None) == 1
    h = lib.vdn_hybrid_attn_fwd_decay
    post = [FAKE, FAKE, None, ctypes.c_float(1e-6), FAKE, None, None, FAKE]
    assert h(ctypes.byref(ok), 0, *pre, None, *post, need, None) == 1
    assert h(ctypes.byref(ok), 0, *pre, MISALIGNED, *post, need, None) == 2
    assert h(ctypes.byref(ok), 0, *pre, FAKE, *post, need - 1, None) == 3


@pytest.fixture(scope="module")
def schedule_dump():
    out = os.path.join(tempfile.mkdtemp(), "schedule_dump")
    src = os.path.join(ROOT, "tests", "host", "schedule_dump.cu")
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    subprocess.run([nvcc, "-std=c++17", "-o", out, src], check=True, capture_output=True)
    return out


def _parse(text, extras=None):
    groups, tiles = [], []
    extent = None
    for line in text.splitlines():
        t = line.split()
        if extras is not None and t[0] == "keytiles":
            extras.setdefault(t[0], {})[int(t[1])] = t[2:]
            continue
        if t[0] == "qsrc":
            groups[int(t[1])]["qsrc"] = int(t[2])
            continue
        if t[0] == "extent":
            extent = (int(t[1]), int(t[2]), int(t[4]))
        elif t[0] == "group":
            segs = [tuple(map(int, s.split(":"))) for s in t[13:]]
            groups.append(dict(g=int(t[1]), q0=int(t[3]), nq=int(t[5]), chunk=int(t[7]),
                               fwd=int(t[9]), rev=int(t[11]), segs=segs))
        elif t[0] == "tile":
            tiles.append((int(t[3]), int(t[5])))
    return extent, groups, tiles


@pytest.mark.parametrize("F", [1, 2, 3, 4, 5, 7, 8, 11, 16, 21, 36])
@pytest.mark.parametrize("c", [1, 2, 3, 5, 6])
def test_cuda_schedule_matches_oracle_key_sets(schedule_dump, F, c):
    N, rows = 3, 4
    r = subprocess.run([schedule_dump, str(F), str(N), str(c), str(rows)], check=True,
                       capture_output=True, text=True)
    (fwd_max, rev_min, ntiles), groups, tiles = _parse(r.stdout)
    covered = []
    need_fwd, need_rev = 0, F - 1
    for G in groups:
        if G["nq"] == 0:
            continue
        assert G["qsrc"] == 0          # no context rows without the joint bits
        frames = sorted({t // N for t in range(G["q0"], G["q0"] + G["nq"])})
        covered += list(range(G["q0"], G["q0"] + G["nq"]))
        key_tokens = set()
        for s0, sn in G["segs"]:
            seg = set(range(s0, s0 + sn))
            assert not (seg & key_tokens), "segments overlap"
            key_tokens |= seg
        for f in frames:
            want = {g * N + n for g in O.softmax_key_frames(f, F, c) for n in range(N)}
            assert key_tokens == want, (F, c, f)
            fr, rr = O.forward_region(f, F, c), O.reverse_region(f, F, c)
            if O.is_boundary(f, F):
                assert G["chunk"] == -1 and len(frames) == 1
                continue
            assert G["chunk"] == O.chunk_of(f, c)
            assert G["fwd"] == (max(fr) if fr else 0)
            assert G["rev"] == (min(rr) if rr else F - 1)
            need_fwd = max(need_fwd, G["fwd"])
            need_rev = min(need_rev, G["rev"])
    assert sorted(covered) == list(range(F * N))
    assert (fwd_max, rev_min) == (need_fwd, need_rev)
    # tiles: every query row in exactly one tile of its group
    seen = []
    for g, r0 in tiles:
        G = groups[g]
        assert G["q0"] <= r0 < G["q0"] + G["nq"]
        seen += [t for t in range(r0, min(r0 + rows, G["q0"] + G["nq"]))]
    assert sorted(seen) == list(range(F * N)) and len(tiles) == ntiles


@pytest.mark.parametrize("F,c,N,T", [(7, 2, 70, 130), (36, 5, 100, 64), (3, 1, 50, 0), (1, 3, 200, 7)])
def test_key_tiles_cover_segments_exactly(schedule_dump, F, c, N, T):
    """128-key tiles of the window kernel: video segments in order, then text;
    every key of the group's key set appears in exactly one tile, only the last
    tile of a segment is partial."""
    r = subprocess.run([schedule_dump, str(F), str(N), str(c), "4"], check=True, capture_output=True,
                       text=True)
    # the dump uses T = 1; rerun the parse with our own T through the oracle's key set
    extras = {}
    _, groups, _ = _parse(r.stdout, extras)
    for G in groups:
        if G["nq"] == 0:
            continue
        tiles = [tuple(map(int, x.split(":"))) for x in extras["keytiles"][G["g"]]]
        video = [(row, valid) for src, row, valid in tiles if src == 0]
        text_tiles = [(row, valid) for src, row, valid in tiles if src == 1]
        keys = []
        for row, valid in video:
            assert 1 <= valid <= 128
            keys += list(range(row, row + valid))
        assert sorted(keys) == sorted(k for s0, sn in G["segs"] for k in range(s0, s0 + sn))
        assert len(keys) == len(set(keys))
        assert [v for _, v in text_tiles] == [1]  # the dump program uses one text token




@pytest.mark.parametrize("F,c,N,T,A,ctx", [(7, 2, 70, 130, 203, 3), (36, 5, 100, 64, 1, 1),
                                           (3, 1, 50, 0, 129, 2), (1, 3, 200, 7, 0, 3),
                                           (12, 2, 1, 2, 5, 3)])
def test_joint_schedule_context_groups_and_audio_tiles(schedule_dump, F, c, N, T, A, ctx):
    """Joint layer: the text/audio query rows are groups scheduled before every
    video group, each row in exactly one tile, with every video token as keys;
    every group's key tiles are its video segments, then the text, then the
    audio, each key once."""
    rows = 4
    r = subprocess.run([schedule_dump, str(F), str(N), str(c), str(rows), str(T), str(A), str(ctx)],
                       check=True, capture_output=True, text=True)
    extras = {}
    (_, _, ntiles), groups, tiles = _parse(r.stdout, extras)
    want_rows = {1: T if ctx & 1 else 0, 2: A if ctx & 2 else 0}
    for src in (1, 2):
        gs = [G for G in groups if G["qsrc"] == src]
        assert len(gs) == 1 and gs[0]["nq"] == want_rows[src] and gs[0]["q0"] == 0
        assert gs[0]["segs"] == [(0, F * N)] and gs[0]["chunk"] == -1
    # schedule order: all context tiles come first, every row once
    first_video = next(i for i, (g, _) in enumerate(tiles) if groups[g]["qsrc"] == 0)
    assert all(groups[g]["qsrc"] != 0 for g, _ in tiles[:first_video])
    assert all(groups[g]["qsrc"] == 0 for g, _ in tiles[first_video:])
    for src in (1, 2):
        seen = []
        for g, r0 in tiles:
            if groups[g]["qsrc"] == src:
                seen += list(range(r0, min(r0 + rows, want_rows[src])))
        assert sorted(seen) == list(range(want_rows[src]))
    video_rows = []
    for g, r0 in tiles:
        G = groups[g]
        if G["qsrc"] == 0:
            video_rows += list(range(r0, min(r0 + rows, G["q0"] + G["nq"])))
    assert sorted(video_rows) == list(range(F * N)) and len(tiles) == ntiles
    for G in groups:
        if G["nq"] == 0:
            continue
        kt = [tuple(map(int, x.split(":"))) for x in extras["keytiles"][G["g"]]]
        srcs = [s for s, _, _ in kt]
        assert srcs == sorted(srcs)     # video, then text, then audio
        for src, n, segs in ((0, None, G["segs"]), (1, T, [(0, T)]), (2, A, [(0, A)])):
            keys = []
            for s, row, valid in kt:
                if s == src:
                    assert 1 <= valid <= 128
                    keys += list(range(row, row + valid))
            assert keys == [k for s0, sn in segs for k in range(s0, s0 + sn)]


def _ctx(lib, **kw):
    from linear_attention_video_block_b200 import vdn
    base = dict(A=0, k_audio=None, v_audio=None, q_text=None, q_audio=None, o_text=None,
                o_audio=None, lse_text=None, lse_audio=None)
    base.update(kw)
    return vdn._CContext(base["A"], *[base[k] for k in ("k_audio", "v_audio", "q_text", "q_audio",
                                                         "o_text", "o_audio", "lse_text", "lse_audio")])


def test_joint_entries_validate_context(lib):
    """vdn_joint_softmax_fwd / vdn_joint_attn_fwd: the context struct is required;
    audio tensors are required when A > 0, outputs with their query rows, every
    given pointer 16-byte aligned (no GPU is touched by any of these)."""
    ok = _layout()
    js = lib.vdn_joint_softmax_fwd
    args = [FAKE] * 6 + [None, None]
    assert js(ctypes.byref(ok), 0, None, *args) == 1
    assert js(ctypes.byref(ok), 0, ctypes.byref(_ctx(lib, A=-1)), *args) == 1
    assert js(ctypes.byref(ok), 0, ctypes.byref(_ctx(lib, A=3)), *args) == 1            # no audio k/v
    assert js(ctypes.byref(ok), 0, ctypes.byref(_ctx(lib, A=3, k_audio=FAKE, v_audio=MISALIGNED)),
              *args) == 2
    assert js(ctypes.byref(ok), 0, ctypes.byref(_ctx(lib, q_text=FAKE)), *args) == 1     # no o_text
    assert js(ctypes.byref(ok), 0, ctypes.byref(_ctx(lib, q_text=FAKE, o_text=MISALIGNED)),
              *args) == 2
    assert js(ctypes.byref(ok), 0, ctypes.byref(_ctx(lib, A=2, k_audio=FAKE, v_audio=FAKE,
                                                     q_audio=FAKE)), *args) == 1         # no o_audio
    assert js(ctypes.byref(_layout(B=0)), 0, ctypes.byref(_ctx(lib)), *args) == 1
    ja = lib.vdn_joint_attn_fwd
    need = lib.vdn_workspace_bytes(ctypes.byref(ok), 0)
    pre = [FAKE] * 7
    post = [None, FAKE, FAKE, None, ctypes.c_float(1e-6), FAKE, None, None, FAKE]
    assert ja(ctypes.byref(ok), 0, None, *pre, *post, need, None) == 1
    assert ja(ctypes.byref(ok), 0, ctypes.byref(_ctx(lib, A=1)), *pre, *post, need, None) == 1
    assert ja(ctypes.byref(ok), 0, ctypes.byref(_ctx(lib)), *pre, *post, need - 1, None) == 3
    assert ja(ctypes.byref(ok), 0, ctypes.byref(_ctx(lib)), *pre, MISALIGNED, *post[1:], need,
              None) == 2                                                                  # alpha


def test_fp8_entry_validates(lib):
    """vdn_window_softmax_fwd_fp8: d = 128 only, positive finite scales, required
    pointers, 16-byte alignment (no GPU is touched)."""
    f = lib.vdn_window_softmax_fwd_fp8
    F = ctypes.c_float
    ok = _layout(d=128)
    args = [FAKE] * 5
    assert f(ctypes.byref(_layout(d=64)), *args, F(1), F(1), F(1), FAKE, None, None) == 2
    assert f(ctypes.byref(ok), *args, F(0), F(1), F(1), FAKE, None, None) == 1
    assert f(ctypes.byref(ok), *args, F(1), F(-1), F(1), FAKE, None, None) == 1
    assert f(ctypes.byref(ok), *args, F(1), F(1), F(float("inf")), FAKE, None, None) == 1
    assert f(ctypes.byref(ok), *args, F(1), F(1), F(1), None, None, None) == 1
    assert f(ctypes.byref(ok), MISALIGNED, *args[1:], F(1), F(1), F(1), FAKE, None, None) == 2
    assert f(ctypes.byref(_layout(d=128, B=0)), *args, F(1), F(1), F(1), FAKE, None, None) == 1


def test_host_pipeline_entry_validates(lib):
    """vdn_hybrid_attn_fwd_host rejects before any copy or launch."""
    f = lib.vdn_hybrid_attn_fwd_host
    ok = _layout()
    need = lib.vdn_hybrid_host_workspace_bytes(ctypes.byref(ok), 0, 0)
    assert need > lib.vdn_workspace_bytes(ctypes.byref(ok), 0)
    args = [FAKE] * 9 + [None, ctypes.c_float(1e-6), FAKE, FAKE]
    assert f(ctypes.byref(_layout(B=0)), 0, 0, *args, need) == 1
    assert f(ctypes.byref(_layout(d=48)), 0, 0, *args, need) == 2
    assert f(ctypes.byref(ok), 5, 0, *args, need) == 2
    assert f(ctypes.byref(ok), 0, 0, *args, need - 1) == 3
    assert f(ctypes.byref(ok), 0, 0, None, *args[1:], need) == 1
    assert f(ctypes.byref(ok), 0, 0, *args[:10], ctypes.c_float(-1.0), FAKE, FAKE, need) == 1


# ------------------------------------------------------ binding validation
# The kernels derive every address from the layout (TMA tensor maps, token
# offsets), so the Python binding checks each tensor's shape, dtype and device
# against the layout before the library is touched. These run on the CPU: a
# well-formed call gets as far as the "needs a CUDA device" check, and a
# mis-sized argument is refused before that.

def _binding_inputs(layout, dtype):
    import torch
    from linear_attention_video_block_b200.synth import make_inputs
    inp = make_inputs(layout, dtype, 5)
    J = -(-layout.F // layout.c)
    extra = {
        "alpha": torch.ones((layout.B, layout.F, layout.H, layout.d)),
        "rms_weight": torch.ones(layout.d),
        "chunk_states": torch.zeros((layout.B, layout.H, 2, J, layout.d, layout.d)),
        "lse": torch.zeros((layout.B, layout.L, layout.H)),
        "out": torch.empty_like(inp["q"]),
    }
    return inp, extra


@pytest.fixture
def no_library(monkeypatch):
    from linear_attention_video_block_b200 import vdn

    def refuse():
        raise AssertionError("the library was reached")
    monkeypatch.setattr(vdn, "lib", refuse)
    return vdn


def _calls(vdn, layout, inp, extra, bad):
    """The public calls with argument `bad` = (name, tensor) substituted."""
    a = dict(inp, **extra)
    if bad is not None:
        a[bad[0]] = bad[1]
    L = layout
    return {
        "window_softmax_fwd": lambda: vdn.window_softmax_fwd(
            L, a["q"], a["k"], a["v"], a["k_text"], a["v_text"], o_soft=a.get("o_soft"), lse=a["lse"]),
        "vda_scan_fwd": lambda: vdn.vda_scan_fwd(
            L, a["q"], a["k"], a["v"], a["k_text"], a["v_text"], a["beta"], a["beta_text"],
            chunk_states=a["chunk_states"], alpha=a["alpha"]),
        "hybrid_attn_fwd": lambda: vdn.hybrid_attn_fwd(
            L, a["q"], a["k"], a["v"], a["k_text"], a["v_text"], a["beta"], a["beta_text"], a["g_s"],
            a["g_l"], rms_weight=a["rms_weight"], out=a["out"]),
        "vda_scan_fwd_noalloc": lambda: vdn.vda_scan_fwd_noalloc(
            L, a["q"], a["k"], a["v"], a["k_text"], a["v_text"], a["beta"], a["beta_text"], a["out"],
            chunk_states=a["chunk_states"]),
    }


BAD_ARGS = [
    # (argument, how it is made wrong, calls that take it)
    ("q", "short", ["window_softmax_fwd", "vda_scan_fwd", "hybrid_attn_fwd", "vda_scan_fwd_noalloc"]),
    ("k", "short", ["window_softmax_fwd", "vda_scan_fwd", "hybrid_attn_fwd", "vda_scan_fwd_noalloc"]),
    ("v", "heads", ["window_softmax_fwd", "vda_scan_fwd", "hybrid_attn_fwd", "vda_scan_fwd_noalloc"]),
    ("k_text", "short", ["window_softmax_fwd", "vda_scan_fwd", "hybrid_attn_fwd", "vda_scan_fwd_noalloc"]),
    ("v_text", "dtype", ["window_softmax_fwd", "vda_scan_fwd", "hybrid_attn_fwd", "vda_scan_fwd_noalloc"]),
    ("beta", "dtype", ["vda_scan_fwd", "hybrid_attn_fwd", "vda_scan_fwd_noalloc"]),
    ("beta", "short", ["vda_scan_fwd", "hybrid_attn_fwd", "vda_scan_fwd_noalloc"]),
    ("beta_text", "short", ["vda_scan_fwd", "hybrid_attn_fwd", "vda_scan_fwd_noalloc"]),
    ("beta_text", "none", ["vda_scan_fwd", "hybrid_attn_fwd", "vda_scan_fwd_noalloc"]),
    ("g_s", "short", ["hybrid_attn_fwd"]),
    ("g_l", "dtype", ["hybrid_attn_fwd"]),
    ("alpha", "short", ["vda_scan_fwd"]),
    ("rms_weight", "short", ["hybrid_attn_fwd"]),
    ("chunk_states", "short", ["vda_scan_fwd", "vda_scan_fwd_noalloc"]),
    ("lse", "short", ["window_softmax_fwd"]),
    ("out", "short", ["hybrid_attn_fwd", "vda_scan_fwd_noalloc"]),
    ("q", "noncontiguous", ["window_softmax_fwd", "hybrid_attn_fwd"]),
]


def _spoil(t, how):
    import torch
    if how == "none":
        return None
    if how == "short":
        return t.reshape(-1)[: t.numel() - 1].clone() if t.dim() == 1 else t[..., :-1, :].clone() \
            if t.dim() >= 2 and t.shape[-2] > 1 else t[..., :-1].clone()
    if how == "heads":
        return torch.cat([t, t[:, :, :1]], dim=2)
    if how == "dtype":
        return t.to(torch.float16)
    if how == "noncontiguous":
        return t.transpose(1, 2).contiguous().transpose(1, 2)
    raise ValueError(how)


@pytest.mark.parametrize("name,how,calls", BAD_ARGS, ids=[f"{a}-{b}" for a, b, _ in BAD_ARGS])
def test_binding_refuses_mis_sized_arguments_before_the_library(no_library, name, how, calls):
    from linear_attention_video_block_b200.synth import Layout
    layout = Layout(B=1, F=7, N=24, T=5, c=2, H=3, d=64)
    inp, extra = _binding_inputs(layout, "bf16")
    base = dict(inp, **extra)
    bad = _spoil(base[name], how)
    for call in calls:
        with pytest.raises((ValueError, TypeError)):
            _calls(no_library, layout, inp, extra, (name, bad))[call]()


def test_binding_well_formed_calls_reach_the_device_check(no_library):
    """The same calls with every argument well-formed pass validation and stop
    only at the missing CUDA device (this host has none)."""
    import torch
    from linear_attention_video_block_b200.synth import Layout
    layout = Layout(B=1, F=7, N=24, T=5, c=2, H=3, d=64)
    inp, extra = _binding_inputs(layout, "bf16")
    for name, call in _calls(no_library, layout, inp, extra, None).items():
        if torch.cuda.is_available():
            pytest.skip("a CUDA device is present")
        with pytest.raises(RuntimeError, match="CUDA device"):
            call()


def test_binding_checks_joint_and_fp8_tensors(no_library):
    import torch
    from linear_attention_video_block_b200.synth import Layout, make_context
    vdn = no_library
    layout = Layout(B=1, F=7, N=24, T=5, c=2, H=3, d=64)
    inp, _ = _binding_inputs(layout, "bf16")
    cx = make_context(layout, 9, "bf16", 3)
    args = (layout, inp["q"], inp["k"], inp["v"], inp["k_text"], inp["v_text"])
    with pytest.raises(ValueError):  # audio keys without values
        vdn.joint_softmax_fwd(*args, k_audio=cx["k_audio"])
    with pytest.raises(ValueError):  # audio values of another length
        vdn.joint_softmax_fwd(*args, k_audio=cx["k_audio"], v_audio=cx["v_audio"][:, :-1].clone())
    with pytest.raises(ValueError):  # text query rows of another length
        vdn.joint_softmax_fwd(*args, q_text=cx["q_text"][:, :-1].clone())
    with pytest.raises(ValueError):  # audio query rows without audio keys
        vdn.joint_softmax_fwd(*args, q_audio=cx["q_audio"])
    with pytest.raises(TypeError):  # fp8 entry given bf16 operands
        vdn.window_softmax_fwd_fp8(*args, 1.0, 1.0, 1.0)
    e4 = {k: inp[k].to(torch.float8_e4m3fn) for k in ("q", "k", "v", "k_text", "v_text")}
    with pytest.raises(ValueError):  # fp8 output of another shape
        vdn.window_softmax_fwd_fp8(layout, e4["q"], e4["k"], e4["v"], e4["k_text"], e4["v_text"],
                                   1.0, 1.0, 1.0, o_soft=torch.empty(3, dtype=torch.bfloat16))
    if not torch.cuda.is_available():
        with pytest.raises(RuntimeError, match="CUDA device"):
            vdn.joint_softmax_fwd(*args, k_audio=cx["k_audio"], v_audio=cx["v_audio"],
                                  q_text=cx["q_text"], q_audio=cx["q_audio"])
        with pytest.raises(RuntimeError, match="CUDA device"):
            vdn.window_softmax_fwd_fp8(layout, e4["q"], e4["k"], e4["v"], e4["k_text"], e4["v_text"],
                                       1.0, 1.0, 1.0)
