"""Float64 CPU oracle for the Video DeltaNet hybrid video-video attention forward.

TEST INFRASTRUCTURE ONLY. This module is the slow, plain, obviously-correct
statement of what the CUDA path computes. Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline / reference arm of ``bench.py`` may import
it. The product path (the C-ABI library and its Python binding) never imports,
calls or links it, and it never imports the product path.

Sources (web pages; each function cites the passage it restates):
  [VDN]  "Video DeltaNet: Near-Lossless Hybrid Attention for Video Models"
         (project page, openvdn.github.io), sections
         "Local Softmax and Long-Range Linear Memory",
         "Gating the Softmax and Linear Branch Outputs",
         "Video Delta Attention: A Frame-Wise Solution",
         "Stability of the Inherited State",
         "Correlation-Aware Frame Updates".
  [FTP]  "Faster Than It Plays: Video DeltaNet Generates 14 Seconds of 768p Video
         in 11 Seconds" (deepmagic blog), section "Two branches instead of one",
         which carries the only closed form that survived extraction:
         S_t = (S_bar + B)(I + A)^-1.

Notation follows the pages: frames t (here f), c frames per chunk, keys K with
rows k_u, values V with rows v_u, write strengths beta_u, A = K^T Diag(beta) K,
B = V^T Diag(beta) K, state S of shape (d_v, d_k) so that S k ~ v.

Readings of points the pages leave open (the CUDA path uses the same ones):
  R1  Joint objective: min_S 1/2 sum_u beta_u ||S k_u - v_u||^2 + 1/2 ||S - S_bar||_F^2,
      whose stationarity condition S (I + A) = S_bar + B is the printed closed form.
  R2  No decay by default: S_bar = previous state. With a decay (the KDA gate,
      VDN "Video Delta Attention": S_bar = S_{t-1} Diag(alpha)), alpha_f in
      [0, 1]^{d_k} is given per frame, head and key channel and scales the
      columns (key dimension) of the state before frame f is written, in both
      scans; the text init has no decay.
  R3  Chunks: ch(f) = floor(f / c); the last chunk is partial when c does not
      divide F. Window of a non-boundary frame: chunks ch(f)-1 .. ch(f)+1 that
      exist. Boundary frames 0 and F-1 see every frame.
  R4  One softmax normaliser over window + anchor frames + all text keys; a frame
      that is both in the window and an anchor is counted once. Scale 1/sqrt(d).
  R5  Text init: the T text tokens are written as one VDA "frame" into a zero
      state and the resulting state is halved: S0 = 1/2 B_T (I + A_T)^-1, shared
      by the forward and the reverse scan.
  R6  Scanned frames are 1 .. F-2 only (boundary frames are never written).
      Forward state for window [lo, hi] = state after frames 1 .. lo-1 (S0 if
      none); reverse state = state after frames F-2 down to hi+1 (S0 if none).
  R7  Boundary-frame queries have no linear readout (o_lin = 0).
  R8  o_lin = (S_fwd + S_rev) q, no query scaling.
  R9  RMSNorm over d per head, eps = 1e-6, weight 1 unless given.
  R10 Gates are element-wise logits of shape [B, L, H, d] for both branches:
      out = sigmoid(g_s) * o_soft + sigmoid(g_l) * RMSNorm(o_lin).
  R14 Audio and the context query rows (joint attention layer): the video
      queries' softmax also sees every audio token (after the text keys, one
      normaliser); audio is never written into the VDA states (only the text
      prompt is). Text and audio query rows keep the original dense softmax
      over every key of the layer (all video, text and audio tokens), scale
      1/sqrt(d), no gates (the output projections are outside this op)
      [VDN "Local Softmax ...", attention-map paragraph; glonce "Video DeltaNet
      speeds MiniMax H3 video generation 14.5x", key facts].
  Parity unpinned beyond the invariants tested: R5 (beyond "text counted exactly
  once"), R9 constants, R10 granularity.

Tensor layout (numpy float64 arrays):
  q, k, v, g_s, g_l : [B, L, H, d], L = F * N, token index = f * N + n
  k_text, v_text    : [B, T, H, d]
  beta              : [B, L, H];  beta_text : [B, T, H]
  q_text            : [B, T, H, d]  (context query rows, R14)
  q_audio, k_audio, v_audio : [B, A, H, d]
"""

from __future__ import annotations

import numpy as np

RMS_EPS = 1e-6


# ----------------------------------------------------------------------------
# Key-set schedule  [VDN "Local Softmax and Long-Range Linear Memory"]
# ----------------------------------------------------------------------------

def chunk_of(f: int, c: int) -> int:
    """Chunk index of latent frame f: c consecutive frames form one chunk (R3)."""
    return f // c


def is_boundary(f: int, F: int) -> bool:
    """Frames 0 and F-1 are the boundary frames [VDN, 4-way boundary anchors]."""
    return f == 0 or f == F - 1


def window_bounds(f: int, F: int, c: int) -> tuple[int, int]:
    """Inclusive frame range [lo, hi] of the sliding window of a frame.

    Each chunk attends to itself, the previous chunk and the following chunk
    [VDN "Local Softmax ..."]; chunks that do not exist are dropped (R3).
    Boundary frames attend to every frame (4-way anchors), so their window is
    the whole clip.
    """
    if is_boundary(f, F):
        return 0, F - 1
    j = chunk_of(f, c)
    lo = max(0, c * (j - 1))
    hi = min(F - 1, c * (j + 2) - 1)
    return lo, hi


def softmax_key_frames(f: int, F: int, c: int) -> list[int]:
    """Video frames whose tokens query frame f sees in the softmax branch.

    Window frames plus the two anchor frames 0 and F-1, as a set (R4).
    """
    lo, hi = window_bounds(f, F, c)
    return sorted(set(range(lo, hi + 1)) | {0, F - 1})


def forward_region(f: int, F: int, c: int) -> list[int]:
    """Frames summarised by the forward state read by frame f (R6).

    The forward state covers frames before the local window, excluding the
    boundary frames [VDN "Local Softmax ...": regions disjoint, and do not
    include window or boundary frames]. Empty for boundary frames (R7).
    """
    if is_boundary(f, F):
        return []
    lo, _ = window_bounds(f, F, c)
    return list(range(1, lo))


def reverse_region(f: int, F: int, c: int) -> list[int]:
    """Frames summarised by the reverse state read by frame f (R6)."""
    if is_boundary(f, F):
        return []
    _, hi = window_bounds(f, F, c)
    return list(range(hi + 1, F - 1))


def frame_visibility(F: int, c: int, anchors: bool = True) -> np.ndarray:
    """Boolean [F, F] map: entry (f, g) is True when query frame f sees key frame g
    in the softmax branch. With anchors=False only the chunk window is kept and
    boundary frames keep their own chunk window."""
    vis = np.zeros((F, F), dtype=bool)
    for f in range(F):
        if anchors:
            for g in softmax_key_frames(f, F, c):
                vis[f, g] = True
        else:
            j = chunk_of(f, c)
            lo = max(0, c * (j - 1))
            hi = min(F - 1, c * (j + 2) - 1)
            vis[f, lo:hi + 1] = True
    return vis


def token_mask(F: int, N: int, T: int, c: int) -> np.ndarray:
    """Explicit boolean [L, L + T] softmax mask over video keys then text keys.

    Text keys are globally visible to every video query [VDN "Local Softmax ...":
    text tokens remain globally visible to every frame].
    """
    L = F * N
    vis = frame_visibility(F, c, anchors=True)
    mask = np.zeros((L, L + T), dtype=bool)
    for f in range(F):
        for g in range(F):
            if vis[f, g]:
                mask[f * N:(f + 1) * N, g * N:(g + 1) * N] = True
    mask[:, L:] = True
    return mask


# ----------------------------------------------------------------------------
# Softmax branch  [VDN "Local Softmax ...", "Gating ..."]
# ----------------------------------------------------------------------------

def softmax_branch(q, k, v, k_text, v_text, F, N, c, rows=None, heads=None,
                   return_lse=False, k_audio=None, v_audio=None):
    """o_soft = softmax(q K^T / sqrt(d) over the allowed keys) V, one normaliser
    over window + anchors + text (R4), and the audio keys when given (R14).

    A dense masked softmax: for each query frame the boolean mask row is built
    explicitly and disallowed scores are set to -inf before max-subtraction.

    rows  : optional sorted array of video token indices to evaluate (others are
            left as NaN); None means all.
    heads : optional list of heads to evaluate; None means all.
    Returns o_soft [B, L, H, d] (and lse [B, L, H], natural log, if asked).
    """
    Bn, L, H, d = q.shape
    if k_audio is None:
        k_audio = np.zeros((Bn, 0, H, d))
        v_audio = np.zeros((Bn, 0, H, d))
    T = k_text.shape[1] + k_audio.shape[1]     # every globally visible key
    assert L == F * N
    out = np.full(q.shape, np.nan)
    lse = np.full((Bn, L, H), np.nan)
    rows = np.arange(L) if rows is None else np.asarray(rows)
    heads = range(H) if heads is None else heads
    vis = frame_visibility(F, c, anchors=True)
    scale = 1.0 / np.sqrt(d)
    row_frames = rows // N
    for b in range(Bn):
        for h in heads:
            keys = np.concatenate([k[b, :, h, :], k_text[b, :, h, :], k_audio[b, :, h, :]], axis=0)
            vals = np.concatenate([v[b, :, h, :], v_text[b, :, h, :], v_audio[b, :, h, :]], axis=0)
            for f in np.unique(row_frames):
                sel = rows[row_frames == f]
                allowed = np.zeros(L + T, dtype=bool)
                for g in range(F):
                    if vis[f, g]:
                        allowed[g * N:(g + 1) * N] = True
                allowed[L:] = True
                s = (q[b, sel, h, :] @ keys.T) * scale
                s = np.where(allowed[None, :], s, -np.inf)
                m = s.max(axis=1, keepdims=True)
                p = np.exp(s - m)
                z = p.sum(axis=1, keepdims=True)
                out[b, sel, h, :] = (p @ vals) / z
                lse[b, sel, h] = (m + np.log(z))[:, 0]
    return (out, lse) if return_lse else out


def context_rows(q_ctx, k, v, k_text, v_text, k_audio=None, v_audio=None, heads=None,
                 return_lse=False):
    """Text or audio query rows (R14): the dense softmax of the original layer,
    softmax(q K^T / sqrt(d)) V over every video, text and audio key.

    q_ctx: [B, R, H, d] query rows (text or audio). Returns [B, R, H, d] (and
    the natural-log normaliser [B, R, H] if asked); heads outside ``heads``
    are NaN.
    """
    Bn, R, H, d = q_ctx.shape
    if k_audio is None:
        k_audio = np.zeros((Bn, 0, H, d))
        v_audio = np.zeros((Bn, 0, H, d))
    out = np.full(q_ctx.shape, np.nan)
    lse = np.full((Bn, R, H), np.nan)
    heads = range(H) if heads is None else heads
    scale = 1.0 / np.sqrt(d)
    for b in range(Bn):
        for h in heads:
            keys = np.concatenate([k[b, :, h, :], k_text[b, :, h, :], k_audio[b, :, h, :]], axis=0)
            vals = np.concatenate([v[b, :, h, :], v_text[b, :, h, :], v_audio[b, :, h, :]], axis=0)
            for r0 in range(0, R, 256):          # row blocks bound the score matrix
                sl = slice(r0, min(R, r0 + 256))
                s = (q_ctx[b, sl, h, :] @ keys.T) * scale
                m = s.max(axis=1, keepdims=True)
                p = np.exp(s - m)
                z = p.sum(axis=1, keepdims=True)
                out[b, sl, h, :] = (p @ vals) / z
                lse[b, sl, h] = (m + np.log(z))[:, 0]
    return (out, lse) if return_lse else out


# ----------------------------------------------------------------------------
# Video Delta Attention  [VDN "Video Delta Attention: A Frame-Wise Solution",
#                         FTP "Two branches instead of one"]
# ----------------------------------------------------------------------------

def frame_gram(K, V, beta):
    """A = K^T Diag(beta) K (weighted key Gram), B = V^T Diag(beta) K
    (value-key write matrix) for one frame's U tokens [VDN "Video Delta
    Attention": the A and B used by the frame-wise solve].

    K: [U, d_k], V: [U, d_v], beta: [U]. Returns A [d_k, d_k], B [d_v, d_k].
    """
    Kw = K * beta[:, None]
    return K.T @ Kw, V.T @ Kw


def frame_update(S_bar, K, V, beta):
    """One VDA frame update S = (S_bar + B)(I + A)^-1 [FTP closed form; VDN
    "Video Delta Attention": differentiating the joint objective (R1)].

    Solved, not inverted: S (I + A) = S_bar + B  <=>  (I + A)^T S^T = (S_bar + B)^T.
    """
    A, Bm = frame_gram(K, V, beta)
    d_k = A.shape[0]
    rhs = S_bar + Bm
    return np.linalg.solve((np.eye(d_k) + A).T, rhs.T).T


def text_init(K_T, V_T, beta_T, d_v, d_k):
    """Initial state shared by both scans: the text tokens written by the frame
    rule into a zero state, scaled by one half (R5) [VDN "Local Softmax ...":
    text written into both states, each scaled by one half, so the two readouts
    count it exactly once]."""
    if K_T.shape[0] == 0:
        return np.zeros((d_v, d_k))
    return 0.5 * frame_update(np.zeros((d_v, d_k)), K_T, V_T, beta_T)


def decayed(S, alpha_f):
    """S_bar = S Diag(alpha_f): the KDA channel-wise decay of the inherited state
    (VDN "Video Delta Attention"), alpha_f over the key channels (columns)."""
    return S if alpha_f is None else S * alpha_f[None, :]


def scan_states(Kf, Vf, betaf, S0, F, alphaf=None):
    """Forward and reverse VDA recurrences over frames 1 .. F-2 (R6).

    Kf, Vf: [F, N, d] per-frame keys/values of one (b, h); betaf: [F, N];
    alphaf: optional [F, d_k] decay per frame (R2).
    Returns (fwd, rev): fwd[s] = state after frames 1..s (fwd[0] = S0, s <= F-2);
    rev[s] = state after frames F-2 down to s (rev[F-1] = S0, s >= 1).
    """
    a = (lambda f: None) if alphaf is None else (lambda f: alphaf[f])
    fwd = {0: S0}
    S = S0
    for f in range(1, F - 1):
        S = frame_update(decayed(S, a(f)), Kf[f], Vf[f], betaf[f])
        fwd[f] = S
    rev = {F - 1: S0}
    S = S0
    for f in range(F - 2, 0, -1):
        S = frame_update(decayed(S, a(f)), Kf[f], Vf[f], betaf[f])
        rev[f] = S
    return fwd, rev


def read_states(f, F, c, fwd, rev, S0):
    """States read by query frame f: forward state after frames 1..lo-1 and
    reverse state after frames F-2..hi+1; S0 where a region is empty (R6)."""
    lo, hi = window_bounds(f, F, c)
    s_fwd = fwd[lo - 1] if lo - 1 >= 1 else S0
    s_rev = rev[hi + 1] if hi + 1 <= F - 2 else S0
    return s_fwd, s_rev


def linear_branch(q, k, v, k_text, v_text, beta, beta_text, F, N, c, heads=None,
                  return_states=False, alpha=None):
    """VDA branch readout o_lin [B, L, H, d], ungated and before RMSNorm.

    Computed per frame (not per chunk): every non-boundary query frame reads
    its own (S_fwd + S_rev) and o_lin = (S_fwd + S_rev) q (R8); boundary frames
    read nothing (R7). With return_states, also returns per (b, h) the dicts
    (S0, fwd, rev). alpha: optional decay [B, F, H, d] (R2).
    """
    Bn, L, H, d = q.shape
    heads = range(H) if heads is None else heads
    out = np.full(q.shape, np.nan)
    states = {}
    for b in range(Bn):
        for h in heads:
            Kf = k[b, :, h, :].reshape(F, N, d)
            Vf = v[b, :, h, :].reshape(F, N, d)
            bf = beta[b, :, h].reshape(F, N)
            S0 = text_init(k_text[b, :, h, :], v_text[b, :, h, :],
                           beta_text[b, :, h], d, d)
            af = None if alpha is None else alpha[b, :, h, :]
            fwd, rev = scan_states(Kf, Vf, bf, S0, F, af)
            states[(b, h)] = (S0, fwd, rev)
            for f in range(F):
                sl = slice(f * N, (f + 1) * N)
                if is_boundary(f, F):
                    out[b, sl, h, :] = 0.0
                    continue
                s_fwd, s_rev = read_states(f, F, c, fwd, rev, S0)
                out[b, sl, h, :] = q[b, sl, h, :] @ (s_fwd + s_rev).T
    return (out, states) if return_states else out


# ----------------------------------------------------------------------------
# Norm, gates and combine  [VDN "Gating the Softmax and Linear Branch Outputs"]
# ----------------------------------------------------------------------------

def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def rms_norm(x, eps=RMS_EPS, weight=None):
    """RMSNorm over the last axis (head dim d) (R9)."""
    y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return y if weight is None else y * weight


def combine(o_soft, o_lin, g_s, g_l, eps=RMS_EPS, weight=None):
    """Gated sum of the two branches (R10); returns (out, gated_soft, gated_lin)
    where out = gated_soft + gated_lin. The per-branch output projections are
    identity here (their weights are trained parameters, outside this op)."""
    gs = sigmoid(g_s) * o_soft
    gl = sigmoid(g_l) * rms_norm(o_lin, eps, weight)
    return gs + gl, gs, gl


def hybrid(q, k, v, k_text, v_text, beta, beta_text, g_s, g_l, F, N, c,
           rows=None, heads=None, eps=RMS_EPS, weight=None, alpha=None):
    """The whole hybrid video-video attention forward for the given rows/heads.

    Returns dict with out, out_soft (gated), out_lin (gated), o_soft, o_lin.
    Elements outside the requested rows/heads are NaN.
    """
    o_soft = softmax_branch(q, k, v, k_text, v_text, F, N, c, rows=rows, heads=heads)
    o_lin = linear_branch(q, k, v, k_text, v_text, beta, beta_text, F, N, c, heads=heads,
                          alpha=alpha)
    out, gs, gl = combine(o_soft, o_lin, g_s, g_l, eps, weight)
    return {"out": out, "out_soft": gs, "out_lin": gl, "o_soft": o_soft, "o_lin": o_lin}


def joint_attention(q, k, v, k_text, v_text, beta, beta_text, g_s, g_l, F, N, c,
                    q_text=None, q_audio=None, k_audio=None, v_audio=None,
                    rows=None, heads=None, eps=RMS_EPS, weight=None, alpha=None):
    """The attention of one joint text-video-audio layer (R14): video rows take
    the hybrid (softmax branch with text and audio keys, VDA with the text
    init), text and audio query rows the dense softmax.

    Returns the dict of ``hybrid`` plus o_text and o_audio (None when the
    corresponding query rows are not given).
    """
    o_soft = softmax_branch(q, k, v, k_text, v_text, F, N, c, rows=rows, heads=heads,
                            k_audio=k_audio, v_audio=v_audio)
    o_lin = linear_branch(q, k, v, k_text, v_text, beta, beta_text, F, N, c, heads=heads,
                          alpha=alpha)
    out, gs, gl = combine(o_soft, o_lin, g_s, g_l, eps, weight)
    res = {"out": out, "out_soft": gs, "out_lin": gl, "o_soft": o_soft, "o_lin": o_lin,
           "o_text": None, "o_audio": None}
    if q_text is not None:
        res["o_text"] = context_rows(q_text, k, v, k_text, v_text, k_audio, v_audio, heads=heads)
    if q_audio is not None:
        res["o_audio"] = context_rows(q_audio, k, v, k_text, v_text, k_audio, v_audio, heads=heads)
    return res


# ----------------------------------------------------------------------------
# Test aids (not on the hot path): the token and SANA-WM rules the pages
# contrast with VDA [VDN "Video Delta Attention", "Correlation-Aware ..."].
# ----------------------------------------------------------------------------

def delta_rule_gradient_step(S_bar, k, v, beta):
    """Classic token delta rule: one gradient step on 1/2 ||S k - v||^2 with
    learning rate beta: S_bar - beta (S_bar k - v) k^T."""
    return S_bar - beta * np.outer(S_bar @ k - v, k)


def sana_wm_frame_update(S_bar, K, V, beta):
    """SANA-WM frame-parallel delta rule: every token reads the frozen S_bar,
    keys scaled by 1/sqrt(U); S = S_bar - sum_u beta_u (S_bar k^_u - v_u) k^_u^T
    with k^_u = k_u / sqrt(U). Returns (S, K_hat)."""
    U = K.shape[0]
    Kh = K / np.sqrt(U)
    S = S_bar.copy()
    for u in range(U):
        S = S - beta[u] * np.outer(S_bar @ Kh[u] - V[u], Kh[u])
    return S, Kh
