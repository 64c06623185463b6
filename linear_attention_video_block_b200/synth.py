"""Seeded synthetic inputs for the hybrid video-video attention forward.

This module only draws random numbers; it contains none of the attention
arithmetic. Both the CUDA path and the float64 oracle are fed from it.

Recipe (fixed draw order from one ``torch.Generator`` seeded with ``seed``):
  q, k, v           ~ N(0, 1)                   [B, L, H, d], L = F * N
  k_text, v_text    ~ N(0, 1)                   [B, T, H, d]
  beta logits, beta_text logits ~ N(0, 1)       [B, L, H], [B, T, H]
  g_s, g_l          ~ N(0, 1)                   [B, L, H, d]
then: every key row (video and text) is L2-normalised per (token, head) in fp32,
beta = sigmoid(logit), and q/k/v/text/gates are cast to the storage dtype
(beta stays fp32). ``repeated_keys`` sets, for each (frame, head), every key row
of the frame to that frame's first key row (the repeated-evidence ablation).

``make_decay`` draws the optional per-frame, per-key-channel decay alpha
[B, F, H, d] (fp32) from a second generator seeded with ``seed``:
alpha = 1 - 0.2 u with u ~ U[0, 1), i.e. in (0.8, 1], the slow-forgetting range
of a channel-wise decay gate; it leaves ``make_inputs``' draws unchanged.

``make_context`` draws the other tokens of a joint text-video-audio layer from a
third generator seeded with ``seed``: q_text [B, T, H, d], then q_audio,
k_audio, v_audio [B, A, H, d], all ~ N(0, 1), audio keys L2-normalised like the
others. ``audio_tokens(F)`` is the audio length that goes with F latent frames
in the H3 data layout: 575 audio latents (40 per second) beside 102 latent
frames, so A = round(575 F / 102) (203 at F = 36).

The workloads mirror the token grids of the video model the pages describe
(48 x 84 latent grid at 768p, 30 x 52 at 480p-like, chunks of 5 latent frames,
text prompt tokens); no dataset or trained weights are involved.
"""

from __future__ import annotations

from dataclasses import dataclass, asdict

import torch


@dataclass(frozen=True)
class Layout:
    B: int
    F: int
    N: int
    T: int
    c: int
    H: int
    d: int

    @property
    def L(self) -> int:
        return self.F * self.N

    def as_dict(self):
        return asdict(self)


# Named workloads: (layout, storage dtype, seed).
WORKLOADS = {
    "tiny-f32": (Layout(B=1, F=8, N=16, T=4, c=2, H=1, d=16), "f32", 0),
    "small-bf16": (Layout(B=1, F=20, N=256, T=64, c=5, H=4, d=64), "bf16", 1),
    "480p-bf16": (Layout(B=1, F=21, N=1560, T=256, c=5, H=24, d=128), "bf16", 2),
    "768p-bf16": (Layout(B=1, F=36, N=4032, T=512, c=5, H=40, d=128), "bf16", 3),
    "long-bf16": (Layout(B=1, F=90, N=4032, T=512, c=5, H=40, d=128), "bf16", 4),
    # profiling case: the 768p-like token grid with 4 heads (inputs 149 MB per
    # video tensor, above the 126 MB L2, a few GB on the device in total)
    "768p-h4-bf16": (Layout(B=1, F=36, N=4032, T=512, c=5, H=4, d=128), "bf16", 3),
    # profiling case for the linear branch's kernels: 12 heads fill the GPU
    # (420 Gram / inverse CTAs, 192 scan CTAs) with inputs of 446 MB per video
    # tensor, a few GB on the device in total
    "768p-h12-bf16": (Layout(B=1, F=36, N=4032, T=512, c=5, H=12, d=128), "bf16", 3),
}

TORCH_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def _normal(shape, gen, device):
    return torch.randn(shape, generator=gen, dtype=torch.float32, device=device)


def _l2_normalise_(x):
    x.div_(x.norm(dim=-1, keepdim=True).clamp_min_(1e-30))
    return x


def make_inputs(layout: Layout, dtype: str, seed: int, repeated_keys: bool = False,
                device: str = "cpu"):
    """Draw one input set. Returns a dict of tensors on ``device``.

    Values drawn on a CUDA device follow the same recipe but a different random
    stream than on the CPU; parity tests always draw on the CPU.
    """
    B, F, N, T, H, d = layout.B, layout.F, layout.N, layout.T, layout.H, layout.d
    L = F * N
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    st = TORCH_DTYPES[dtype]
    out = {}
    out["q"] = _normal((B, L, H, d), gen, device).to(st)
    k = _l2_normalise_(_normal((B, L, H, d), gen, device))
    if repeated_keys:
        kf = k.view(B, F, N, H, d)
        kf.copy_(kf[:, :, :1].expand_as(kf))
    out["k"] = k.to(st)
    del k
    out["v"] = _normal((B, L, H, d), gen, device).to(st)
    out["k_text"] = _l2_normalise_(_normal((B, T, H, d), gen, device)).to(st)
    out["v_text"] = _normal((B, T, H, d), gen, device).to(st)
    out["beta"] = torch.sigmoid(_normal((B, L, H), gen, device))
    out["beta_text"] = torch.sigmoid(_normal((B, T, H), gen, device))
    out["g_s"] = _normal((B, L, H, d), gen, device).to(st)
    out["g_l"] = _normal((B, L, H, d), gen, device).to(st)
    return out


def make_decay(layout: Layout, seed: int, device: str = "cpu"):
    """Per-frame channel decay alpha [B, F, H, d] float32 in (0.8, 1]."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    u = torch.rand((layout.B, layout.F, layout.H, layout.d), generator=gen,
                   dtype=torch.float32, device=device)
    return 1.0 - 0.2 * u


def audio_tokens(F: int) -> int:
    """Audio tokens beside F latent frames (575 audio latents per 102 frames)."""
    return int(round(575 * F / 102))


def make_context(layout: Layout, A: int, dtype: str, seed: int, device: str = "cpu"):
    """Text query rows and the audio tokens of a joint layer (see module doc)."""
    B, T, H, d = layout.B, layout.T, layout.H, layout.d
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    st = TORCH_DTYPES[dtype]
    out = {}
    out["q_text"] = _normal((B, T, H, d), gen, device).to(st)
    out["q_audio"] = _normal((B, A, H, d), gen, device).to(st)
    out["k_audio"] = _l2_normalise_(_normal((B, A, H, d), gen, device)).to(st)
    out["v_audio"] = _normal((B, A, H, d), gen, device).to(st)
    return out


E4M3_MAX = 448.0


def quantize_e4m3(*tensors):
    """Float8 e4m3 copies of tensors that share one scale (value = e4m3 *
    scale, scale = max |x| / 448 over all of them). Returns ([t8, ...], scale)."""
    amax = max(float(t.float().abs().max()) if t.numel() else 0.0 for t in tensors)
    scale = (amax / E4M3_MAX) if amax > 0 else 1.0
    return [(t.float() / scale).to(torch.float8_e4m3fn) for t in tensors], scale


def as_float64_numpy(inputs):
    """The oracle's view of an input set: every tensor upcast to float64 (bf16
    rounding of the stored inputs is therefore not counted as error)."""
    return {k: t.detach().to("cpu", torch.float64).numpy() for k, t in inputs.items()}
