"""Pins for the float64 oracle: checks against what the pages and the
mathematics fix, never against the oracle's own formula retyped.

Each test names the passage or the mathematical fact it relies on. Together
they are meant to catch a dropped term, a wrong sign, an off-by-one in the
window or the read states, or a transposed operand anywhere in the oracle.
"""

import json
import os

import numpy as np
import pytest
import torch

from oracle import vdn_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _unit_rows(rng, n, d):
    x = rng.standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def _rand_inputs(rng, B, F, N, T, H, d):
    L = F * N
    q = rng.standard_normal((B, L, H, d))
    k = rng.standard_normal((B, L, H, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, L, H, d))
    kt = rng.standard_normal((B, T, H, d))
    if T:
        kt /= np.linalg.norm(kt, axis=-1, keepdims=True)
    vt = rng.standard_normal((B, T, H, d))
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, L, H))))
    bt = 1 / (1 + np.exp(-rng.standard_normal((B, T, H))))
    gs = rng.standard_normal((B, L, H, d))
    gl = rng.standard_normal((B, L, H, d))
    return q, k, v, kt, vt, beta, bt, gs, gl


# ---------------------------------------------------------------- schedule --

def test_anchor_density_matches_printed_value():
    """Project page, 'Local Softmax and Long-Range Linear Memory': the anchors add
    3.57% attention density (chunks of five frames). The frame map gives 3.5755%
    (printed digits truncated); with the text key columns counted in the map the
    token-space figure rounds to 3.57%."""
    g = json.load(open(os.path.join(GOLDEN, "anchor_density.json")))
    F, c, N = g["F"], g["c"], g["N"]
    printed = g["printed_value_percent"]
    added_pairs = (O.frame_visibility(F, c, True).sum() - O.frame_visibility(F, c, False).sum())
    frame_pct = 100 * added_pairs / F ** 2
    assert printed <= frame_pct < printed + 0.01
    for T in g["T_values"]:
        L = F * N
        token_pct = 100 * added_pairs * N * N / (L * (L + T))
        assert round(token_pct, 2) == printed


def test_alternative_chunkings_miss_the_printed_density():
    """The pin above discriminates between chunkings: frame 0 alone and then
    groups of 5, or the two boundary frames left out of the chunking, both land
    outside [3.57, 3.58)."""
    F, c = 102, 5

    def added(chunk):
        J = {}
        for f in range(F):
            J.setdefault(chunk(f), []).append(f)
        win = np.zeros((F, F), bool)
        for f in range(F):
            j = chunk(f)
            for jj in (j - 1, j, j + 1):
                for g in J.get(jj, []):
                    win[f, g] = True
        anc = win.copy()
        anc[:, [0, F - 1]] = True
        anc[[0, F - 1], :] = True
        return 100 * (anc.sum() - win.sum()) / F ** 2

    assert 3.57 <= added(lambda f: f // c) < 3.58
    for alt in (lambda f: 0 if f == 0 else 1 + (f - 1) // c,
                lambda f: -1 if f == 0 else (10 ** 6 if f == F - 1 else (f - 1) // c)):
        assert not (3.57 <= added(alt) < 3.58)


def test_hand_counted_density_small_layout():
    g = json.load(open(os.path.join(GOLDEN, "hand_counts_F8_c2.json")))
    vis = O.frame_visibility(g["F"], g["c"], True)
    assert O.frame_visibility(g["F"], g["c"], False).mean() == g["window_density"]
    assert vis.mean() == g["anchored_density"]
    assert vis.sum(axis=1).tolist() == g["anchored_row_counts"]


@pytest.mark.parametrize("F", list(range(1, 25)))
@pytest.mark.parametrize("c", [1, 2, 3, 4, 5, 6])
def test_regions_partition_every_frame(F, c):
    """Project page, 'Local Softmax ...': forward and reverse regions are disjoint
    and exclude window and boundary frames, so window + anchors + forward +
    reverse cover every frame exactly once for every non-boundary query."""
    for f in range(F):
        keys = set(O.softmax_key_frames(f, F, c))
        if O.is_boundary(f, F):
            assert keys == set(range(F))
            assert O.forward_region(f, F, c) == [] and O.reverse_region(f, F, c) == []
            continue
        fw, rv = set(O.forward_region(f, F, c)), set(O.reverse_region(f, F, c))
        assert not (keys & fw) and not (keys & rv) and not (fw & rv)
        assert keys | fw | rv == set(range(F))
        assert 0 not in fw | rv and F - 1 not in fw | rv
        # forward region strictly before the window, reverse strictly after
        lo, hi = O.window_bounds(f, F, c)
        assert all(g < lo for g in fw) and all(g > hi for g in rv)
        # chunk sharing: all frames of a chunk have the same window
        j = O.chunk_of(f, c)
        for f2 in range(j * c, min(F, (j + 1) * c)):
            if not O.is_boundary(f2, F):
                assert O.window_bounds(f2, F, c) == (lo, hi)


def test_token_mask_counts():
    F, N, T, c = 8, 3, 2, 2
    m = O.token_mask(F, N, T, c)
    vis = O.frame_visibility(F, c)
    assert m.shape == (F * N, F * N + T)
    assert m[:, F * N:].all()
    assert (m[:, :F * N].sum(axis=1) == np.repeat(vis.sum(axis=1) * N, N)).all()


# ---------------------------------------------------------------- softmax ---

def test_softmax_equals_full_attention_when_window_covers_clip():
    """When F <= 2c every chunk window covers the clip, so the branch is plain
    full attention over video + text keys: compare with torch's
    scaled_dot_product_attention in float64."""
    rng = np.random.default_rng(1)
    B, F, N, T, H, d, c = 2, 6, 5, 3, 2, 8, 3
    q, k, v, kt, vt, *_ = _rand_inputs(rng, B, F, N, T, H, d)
    got, lse = O.softmax_branch(q, k, v, kt, vt, F, N, c, return_lse=True)
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(np.concatenate([k, kt], 1)).permute(0, 2, 1, 3)
    tv = torch.from_numpy(np.concatenate([v, vt], 1)).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).permute(0, 2, 1, 3)
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)
    ref_lse = torch.logsumexp(tq @ tk.transpose(-1, -2) / np.sqrt(d), -1).permute(0, 2, 1)
    np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=1e-12, atol=1e-12)


def test_softmax_equals_sdpa_on_gathered_key_subset():
    """For each query frame, the masked branch equals unmasked attention over the
    gathered allowed keys (library routine on the subset). With F = 11, c = 2 the
    windows, anchors and overlaps all occur."""
    rng = np.random.default_rng(2)
    B, F, N, T, H, d, c = 1, 11, 4, 3, 2, 8, 2
    q, k, v, kt, vt, *_ = _rand_inputs(rng, B, F, N, T, H, d)
    got = O.softmax_branch(q, k, v, kt, vt, F, N, c)
    for f in range(F):
        idx = np.concatenate([np.arange(g * N, (g + 1) * N) for g in O.softmax_key_frames(f, F, c)])
        ks = np.concatenate([k[:, idx], kt], 1)
        vs = np.concatenate([v[:, idx], vt], 1)
        tq = torch.from_numpy(q[:, f * N:(f + 1) * N]).permute(0, 2, 1, 3)
        ref = torch.nn.functional.scaled_dot_product_attention(
            tq, torch.from_numpy(ks).permute(0, 2, 1, 3), torch.from_numpy(vs).permute(0, 2, 1, 3))
        np.testing.assert_allclose(got[:, f * N:(f + 1) * N], ref.permute(0, 2, 1, 3).numpy(),
                                   rtol=1e-12, atol=1e-12)


def test_softmax_ignores_keys_outside_the_key_set():
    """Changing k/v of a frame outside K(f) leaves frame f's output unchanged,
    changing one inside changes it."""
    rng = np.random.default_rng(3)
    B, F, N, T, H, d, c = 1, 12, 3, 2, 1, 4, 2
    q, k, v, kt, vt, *_ = _rand_inputs(rng, B, F, N, T, H, d)
    base = O.softmax_branch(q, k, v, kt, vt, F, N, c)
    for g in range(F):
        v2 = v.copy()
        v2[:, g * N:(g + 1) * N] += 1.0
        out = O.softmax_branch(q, k, v2, kt, vt, F, N, c)
        for f in range(F):
            changed = not np.allclose(out[:, f * N:(f + 1) * N], base[:, f * N:(f + 1) * N])
            assert changed == (g in O.softmax_key_frames(f, F, c))


# -------------------------------------------------------------------- VDA ---

def test_single_token_frame_is_sherman_morrison_delta_step():
    """A frame of U = 1 token: (S_bar + beta v k^T)(I + beta k k^T)^-1 equals
    S_bar + beta (v - S_bar k) k^T / (1 + beta ||k||^2) (Sherman-Morrison), the
    implicit form of the token delta rule (project page, 'Video Delta
    Attention'). Unnormalised k so that ||k|| matters."""
    rng = np.random.default_rng(4)
    d_v, d_k = 5, 7
    S_bar = rng.standard_normal((d_v, d_k))
    k = rng.standard_normal(d_k) * 1.7
    v = rng.standard_normal(d_v)
    beta = 0.63
    got = O.frame_update(S_bar, k[None], v[None], np.array([beta]))
    ref = S_bar + beta * np.outer(v - S_bar @ k, k) / (1 + beta * k @ k)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_one_token_frames_scan_equals_token_loop():
    """With N = 1 the forward scan is a token-by-token loop of the implicit delta
    step over frames 1..F-2, starting from the half-weight text state."""
    rng = np.random.default_rng(5)
    B, F, N, T, H, d, c = 1, 9, 1, 3, 1, 6, 2
    q, k, v, kt, vt, beta, bt, *_ = _rand_inputs(rng, B, F, N, T, H, d)
    _, st = O.linear_branch(q, k, v, kt, vt, beta, bt, F, N, c, return_states=True)
    S0, fwd, rev = st[(0, 0)]
    S = S0.copy()
    for f in range(1, F - 1):
        kk, vv, bb = k[0, f, 0], v[0, f, 0], beta[0, f, 0]
        S = S + bb * np.outer(vv - S @ kk, kk) / (1 + bb * kk @ kk)
        np.testing.assert_allclose(fwd[f], S, rtol=1e-11, atol=1e-12)
    S = S0.copy()
    for f in range(F - 2, 0, -1):
        kk, vv, bb = k[0, f, 0], v[0, f, 0], beta[0, f, 0]
        S = S + bb * np.outer(vv - S @ kk, kk) / (1 + bb * kk @ kk)
        np.testing.assert_allclose(rev[f], S, rtol=1e-11, atol=1e-12)


def test_frame_update_is_the_joint_objective_minimiser():
    """Reading R1: the update minimises 1/2 sum beta ||S k - v||^2 + 1/2 ||S -
    S_bar||^2. Check the gradient vanishes and random perturbations increase
    the objective."""
    rng = np.random.default_rng(6)
    U, d = 11, 6
    K = _unit_rows(rng, U, d)
    V = rng.standard_normal((U, d))
    beta = rng.uniform(0, 1, U)
    S_bar = rng.standard_normal((d, d))
    S = O.frame_update(S_bar, K, V, beta)

    def obj(X):
        r = X @ K.T - V.T
        return 0.5 * np.sum(beta * np.sum(r * r, 0)) + 0.5 * np.sum((X - S_bar) ** 2)

    grad = ((S @ K.T - V.T) * beta) @ K + (S - S_bar)
    assert np.abs(grad).max() < 1e-12
    for _ in range(10):
        assert obj(S + 1e-3 * rng.standard_normal(S.shape)) > obj(S)


def test_repeated_keys_closed_form():
    """Project page, 'Correlation-Aware Frame Updates', repeated-key geometry:
    k_u = k (unit) gives S = S_bar + (w - s S_bar k) k^T / (1 + s), s = sum beta,
    w = sum beta_u v_u; with S_bar = 0 and a shared beta, S k = U beta / (1 + U
    beta) * mean(v)."""
    rng = np.random.default_rng(7)
    U, d = 9, 5
    k = _unit_rows(rng, 1, d)[0]
    K = np.tile(k, (U, 1))
    V = rng.standard_normal((U, d))
    beta = rng.uniform(0, 1, U)
    S_bar = rng.standard_normal((d, d))
    s, w = beta.sum(), (beta[:, None] * V).sum(0)
    np.testing.assert_allclose(O.frame_update(S_bar, K, V, beta),
                               S_bar + np.outer(w - s * S_bar @ k, k) / (1 + s), atol=1e-12)
    b = 0.4
    S = O.frame_update(np.zeros((d, d)), K, V, np.full(U, b))
    np.testing.assert_allclose(S @ k, U * b / (1 + U * b) * V.mean(0), atol=1e-12)
    # SANA-WM on the same frame predicts beta * mean(v) whatever U is
    S2, Kh = O.sana_wm_frame_update(np.zeros((d, d)), K, V, np.full(U, b))
    np.testing.assert_allclose(S2 @ Kh[0], b * V.mean(0), atol=1e-12)


def test_orthonormal_keys_closed_form():
    """Project page, 'Correlation-Aware Frame Updates', orthonormal geometry:
    S k_u = (S_bar k_u + beta_u v_u) / (1 + beta_u) and S z = S_bar z for z
    orthogonal to every k_u; SANA-WM gives beta v_u / U on its scaled key."""
    rng = np.random.default_rng(8)
    U, d = 4, 7
    Q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    K = Q[:, :U].T
    V = rng.standard_normal((U, d))
    beta = rng.uniform(0, 1, U)
    S_bar = rng.standard_normal((d, d))
    S = O.frame_update(S_bar, K, V, beta)
    for u in range(U):
        np.testing.assert_allclose(S @ K[u], (S_bar @ K[u] + beta[u] * V[u]) / (1 + beta[u]), atol=1e-12)
    for z in Q[:, U:].T:
        np.testing.assert_allclose(S @ z, S_bar @ z, atol=1e-12)
    b = 0.7
    S2, Kh = O.sana_wm_frame_update(np.zeros((d, d)), K, V, np.full(U, b))
    for u in range(U):
        np.testing.assert_allclose(S2 @ Kh[u], b * V[u] / U, atol=1e-12)


def test_transition_is_non_expansive():
    """Project page, 'Stability of the Inherited State': for A >= 0 the transition
    (I + A)^-1 has eigenvalues 1/(1 + lambda_i(A)) in (0, 1], so
    ||S_bar (I + A)^-1||_2 <= ||S_bar||_2, for any number or alignment of
    tokens; lambda_max(A) <= tr(A) = sum beta for unit keys."""
    rng = np.random.default_rng(9)
    d = 8
    for U, aligned in [(3, False), (50, False), (200, True)]:
        K = _unit_rows(rng, U, d)
        if aligned:
            K = _unit_rows(rng, 1, d) + 0.05 * rng.standard_normal((U, d))
            K /= np.linalg.norm(K, axis=1, keepdims=True)
        beta = rng.uniform(0, 1, U)
        A, _ = O.frame_gram(K, np.zeros((U, d)), beta)
        lam = np.linalg.eigvalsh(A)
        assert lam.min() > -1e-12 and lam.max() <= beta.sum() + 1e-9
        # the inherited-state part of the update is S_bar -> S_bar (I + A)^-1
        # (V = 0 removes the write), so probing with S_bar = I reads the map
        M = O.frame_update(np.eye(d), K, np.zeros((U, d)), beta)
        np.testing.assert_allclose(np.sort(np.linalg.eigvalsh((M + M.T) / 2)),
                                   np.sort(1 / (1 + lam)), atol=1e-10)
        assert np.linalg.norm(M, 2) <= 1 + 1e-12
        for _ in range(5):
            Sb = rng.standard_normal((d, d))
            assert np.linalg.norm(O.frame_update(Sb, K, np.zeros((U, d)), beta), 2) <= \
                np.linalg.norm(Sb, 2) + 1e-12
        if aligned:  # the additive transition I - A is expansive here
            assert np.abs(1 - lam).max() > 1


def test_neumann_first_order():
    """Project page, 'Correlation-Aware Frame Updates': (I + A)^-1 = I - A + A^2 -
    ..., so S_bar (I + eps A)^-1 - S_bar (I - eps A) = O(eps^2)."""
    rng = np.random.default_rng(10)
    U, d = 6, 5
    K = _unit_rows(rng, U, d)
    beta = rng.uniform(0, 1, U)
    S_bar = rng.standard_normal((d, d))
    A, _ = O.frame_gram(K, np.zeros((U, d)), beta)
    ratios = []
    for eps in [1e-2, 1e-3]:
        got = O.frame_update(S_bar, K, np.zeros((U, d)), eps * beta)
        r = np.abs(got - S_bar @ (np.eye(d) - eps * A)).max()
        second = np.abs(S_bar @ (eps * A) @ (eps * A)).max()
        ratios.append(r / second)
    assert all(0.5 < x < 2.0 for x in ratios)


def test_solve_matches_inverse_and_eigen_form():
    rng = np.random.default_rng(11)
    U, d = 30, 6
    K = _unit_rows(rng, U, d)
    V = rng.standard_normal((U, d))
    beta = rng.uniform(0, 1, U)
    S_bar = rng.standard_normal((d, d))
    A, Bm = O.frame_gram(K, V, beta)
    lam, Qm = np.linalg.eigh(A)
    ref = (S_bar + Bm) @ Qm @ np.diag(1 / (1 + lam)) @ Qm.T
    np.testing.assert_allclose(O.frame_update(S_bar, K, V, beta), ref, atol=1e-11)
    np.testing.assert_allclose(O.frame_update(S_bar, K, V, beta),
                               (S_bar + Bm) @ np.linalg.inv(np.eye(d) + A), atol=1e-11)


def test_gram_orientation():
    """A = K^T Diag(beta) K and B = V^T Diag(beta) K entry by entry, with d_v != d_k
    so a transposed operand cannot pass."""
    rng = np.random.default_rng(12)
    U, dk, dv = 4, 3, 5
    K = rng.standard_normal((U, dk))
    V = rng.standard_normal((U, dv))
    beta = rng.uniform(0, 1, U)
    A, Bm = O.frame_gram(K, V, beta)
    assert A.shape == (dk, dk) and Bm.shape == (dv, dk)
    for i in range(dk):
        for j in range(dk):
            assert abs(A[i, j] - sum(beta[u] * K[u, i] * K[u, j] for u in range(U))) < 1e-12
    for i in range(dv):
        for j in range(dk):
            assert abs(Bm[i, j] - sum(beta[u] * V[u, i] * K[u, j] for u in range(U))) < 1e-12


# ------------------------------------------------------- linear branch wiring

def test_text_counted_exactly_once():
    """Project page, 'Local Softmax ...': with no video writes (beta = 0 on video),
    the summed readout of every non-boundary frame is the text written once:
    o_lin = (B_T (I + A_T)^-1) q; boundary frames read nothing."""
    rng = np.random.default_rng(13)
    B, F, N, T, H, d, c = 1, 13, 3, 5, 2, 6, 2
    q, k, v, kt, vt, beta, bt, *_ = _rand_inputs(rng, B, F, N, T, H, d)
    beta[:] = 0.0
    o = O.linear_branch(q, k, v, kt, vt, beta, bt, F, N, c)
    for h in range(H):
        A, Bm = O.frame_gram(kt[0, :, h], vt[0, :, h], bt[0, :, h])
        St = Bm @ np.linalg.inv(np.eye(d) + A)
        for f in range(F):
            sl = slice(f * N, (f + 1) * N)
            ref = 0 * q[0, sl, h] if O.is_boundary(f, F) else q[0, sl, h] @ St.T
            np.testing.assert_allclose(o[0, sl, h], ref, atol=1e-12)


def test_each_frame_reaches_a_query_through_exactly_one_branch():
    """Key frame g influences query frame f's linear readout iff g lies in f's
    forward or reverse region, and its softmax output iff g is in the key set:
    together, exactly once for every (f, g) with f non-boundary."""
    rng = np.random.default_rng(14)
    B, F, N, T, H, d, c = 1, 14, 2, 2, 1, 4, 2
    q, k, v, kt, vt, beta, bt, *_ = _rand_inputs(rng, B, F, N, T, H, d)
    beta0 = np.zeros_like(beta)
    base = O.linear_branch(q, k, v, kt, vt, beta0, bt, F, N, c)
    for g in range(F):
        b1 = beta0.copy()
        b1[:, g * N:(g + 1) * N] = 0.9
        o = O.linear_branch(q, k, v, kt, vt, b1, bt, F, N, c)
        for f in range(F):
            sl = slice(f * N, (f + 1) * N)
            lin = not np.allclose(o[:, sl], base[:, sl], atol=1e-13)
            soft = g in O.softmax_key_frames(f, F, c)
            if O.is_boundary(f, F):
                assert soft and not lin
            else:
                assert lin != soft, (f, g)


@pytest.mark.parametrize("F,c", [(12, 3), (10, 2), (8, 4)])
def test_time_reversal_symmetry(F, c):
    """When c divides F the chunking is symmetric, so reversing the frame order of
    every input reverses the output (forward and reverse scans swap roles)."""
    rng = np.random.default_rng(15)
    B, N, T, H, d = 1, 3, 2, 1, 5
    q, k, v, kt, vt, beta, bt, gs, gl = _rand_inputs(rng, B, F, N, T, H, d)

    def rev(x):
        s = x.shape
        return x.reshape(s[0], F, N, *s[2:])[:, ::-1].reshape(s)

    a = O.hybrid(q, k, v, kt, vt, beta, bt, gs, gl, F, N, c)["out"]
    b = O.hybrid(rev(q), rev(k), rev(v), kt, vt, rev(beta), bt, rev(gs), rev(gl), F, N, c)["out"]
    np.testing.assert_allclose(rev(b), a, atol=1e-11)


# --------------------------------------------------------- norm and gates ---

def test_rms_norm_matches_torch():
    rng = np.random.default_rng(16)
    x = rng.standard_normal((3, 7, 2, 16))
    w = rng.standard_normal(16)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (16,), torch.from_numpy(w), eps=1e-6)
    np.testing.assert_allclose(O.rms_norm(x, 1e-6, w), ref.numpy(), rtol=1e-12, atol=1e-12)


def test_gates_select_branches():
    """Project page, 'Gating ...': each branch passes through its own sigmoid gate;
    a closed gate removes that branch, an open one passes it."""
    rng = np.random.default_rng(17)
    o_s = rng.standard_normal((1, 4, 1, 8))
    o_l = rng.standard_normal((1, 4, 1, 8))
    big = np.full(o_s.shape, 60.0)
    out, gs, gl = O.combine(o_s, o_l, big, -big)
    np.testing.assert_allclose(out, o_s, atol=1e-12)
    out, gs, gl = O.combine(o_s, o_l, -big, big)
    np.testing.assert_allclose(out, o_l / np.sqrt(np.mean(o_l ** 2, -1, keepdims=True) + 1e-6), atol=1e-12)
    out, gs, gl = O.combine(o_s, o_l, 0 * big, 0 * big)
    np.testing.assert_allclose(out, gs + gl, atol=0)
    np.testing.assert_allclose(gs, 0.5 * o_s, atol=1e-15)


def test_boundary_frames_have_no_linear_readout():
    rng = np.random.default_rng(18)
    B, F, N, T, H, d, c = 1, 7, 2, 2, 1, 4, 3
    q, k, v, kt, vt, beta, bt, gs, gl = _rand_inputs(rng, B, F, N, T, H, d)
    r = O.hybrid(q, k, v, kt, vt, beta, bt, gs, gl, F, N, c)
    assert np.all(r["o_lin"][:, :N] == 0) and np.all(r["o_lin"][:, -N:] == 0)
    np.testing.assert_allclose(r["out"][:, :N], (1 / (1 + np.exp(-gs)) * r["o_soft"])[:, :N])


@pytest.mark.parametrize("F", [1, 2, 3])
def test_degenerate_clip_lengths(F):
    """F <= 2: every frame is a boundary frame (no scan, no linear readout);
    F = 3: the only scanned frame is 1 and it lies in frame 1's own window."""
    rng = np.random.default_rng(19)
    B, N, T, H, d, c = 1, 3, 2, 1, 4, 5
    q, k, v, kt, vt, beta, bt, gs, gl = _rand_inputs(rng, B, F, N, T, H, d)
    r = O.hybrid(q, k, v, kt, vt, beta, bt, gs, gl, F, N, c)
    assert np.isfinite(r["out"]).all()
    if F <= 2:
        assert np.all(r["o_lin"] == 0)


def test_no_text_tokens():
    """T = 0: the text init is the zero state and the softmax sees video only."""
    rng = np.random.default_rng(20)
    B, F, N, T, H, d, c = 1, 9, 2, 0, 1, 4, 2
    q, k, v, kt, vt, beta, bt, gs, gl = _rand_inputs(rng, B, F, N, T, H, d)
    r = O.hybrid(q, k, v, kt, vt, beta, bt, gs, gl, F, N, c)
    assert np.isfinite(r["out"]).all()
    _, st = O.linear_branch(q, k, v, kt, vt, beta, bt, F, N, c, return_states=True)
    assert np.all(st[(0, 0)][0] == 0)


# ------------------------------------------------ KDA channel decay (option)

def test_decay_without_writes_is_a_product_of_diagonals():
    """With every write strength zero (A = B = 0) the update reduces to the decay
    alone: the forward state after frames 1..f is S0 Diag(prod_{g<=f} alpha_g),
    the reverse one after F-2..f is S0 Diag(prod_{g>=f} alpha_g) (the decay acts on
    the key channels, the columns of S)."""
    rng = np.random.default_rng(30)
    B, F, N, T, H, d, c = 1, 9, 3, 4, 1, 5, 2
    q, k, v, kt, vt, beta, bt, *_ = _rand_inputs(rng, B, F, N, T, H, d)
    beta[:] = 0.0
    alpha = rng.uniform(0.3, 1.0, (B, F, H, d))
    _, st = O.linear_branch(q, k, v, kt, vt, beta, bt, F, N, c, return_states=True, alpha=alpha)
    S0, fwd, rev = st[(0, 0)]
    for f in range(1, F - 1):
        np.testing.assert_allclose(fwd[f], S0 * np.prod(alpha[0, 1:f + 1, 0], axis=0)[None, :], atol=1e-13)
        np.testing.assert_allclose(rev[f], S0 * np.prod(alpha[0, f:F - 1, 0], axis=0)[None, :], atol=1e-13)


def test_decay_one_token_frames_match_the_decayed_delta_step():
    """One-token frames with decay: S <- S_bar + beta (v - S_bar k) k^T / (1 + beta |k|^2)
    with S_bar = S Diag(alpha_f), frame by frame (Sherman-Morrison again)."""
    rng = np.random.default_rng(31)
    B, F, N, T, H, d, c = 1, 8, 1, 2, 1, 6, 2
    q, k, v, kt, vt, beta, bt, *_ = _rand_inputs(rng, B, F, N, T, H, d)
    alpha = rng.uniform(0.5, 1.0, (B, F, H, d))
    _, st = O.linear_branch(q, k, v, kt, vt, beta, bt, F, N, c, return_states=True, alpha=alpha)
    S0, fwd, _ = st[(0, 0)]
    S = S0.copy()
    for f in range(1, F - 1):
        Sb = S @ np.diag(alpha[0, f, 0])
        kk, vv, bb = k[0, f, 0], v[0, f, 0], beta[0, f, 0]
        S = Sb + bb * np.outer(vv - Sb @ kk, kk) / (1 + bb * kk @ kk)
        np.testing.assert_allclose(fwd[f], S, rtol=1e-11, atol=1e-12)


def test_decay_keeps_the_transition_non_expansive():
    """Project page, 'Stability of the Inherited State': with 0 <= alpha <= 1 the
    inherited component passes through Diag(alpha)(I + A)^-1, of norm <= 1."""
    rng = np.random.default_rng(32)
    d, U = 7, 40
    K = _unit_rows(rng, U, d)
    beta = rng.uniform(0, 1, U)
    for _ in range(5):
        alpha = rng.uniform(0, 1, d)
        Sb = rng.standard_normal((d, d))
        out = O.frame_update(O.decayed(Sb, alpha), K, np.zeros((U, d)), beta)
        assert np.linalg.norm(out, 2) <= np.linalg.norm(Sb, 2) + 1e-12


def test_unit_decay_is_no_decay():
    rng = np.random.default_rng(33)
    B, F, N, T, H, d, c = 1, 10, 2, 3, 2, 4, 3
    q, k, v, kt, vt, beta, bt, gs, gl = _rand_inputs(rng, B, F, N, T, H, d)
    a = O.hybrid(q, k, v, kt, vt, beta, bt, gs, gl, F, N, c)["out"]
    b = O.hybrid(q, k, v, kt, vt, beta, bt, gs, gl, F, N, c, alpha=np.ones((B, F, H, d)))["out"]
    np.testing.assert_array_equal(a, b)


# ---------------------------------------------- joint layer: audio, context rows ---

def _rand_context(rng, B, T, A, H, d):
    qt = rng.standard_normal((B, T, H, d))
    qa = rng.standard_normal((B, A, H, d))
    ka = rng.standard_normal((B, A, H, d))
    if A:
        ka /= np.linalg.norm(ka, axis=-1, keepdims=True)
    va = rng.standard_normal((B, A, H, d))
    return qt, qa, ka, va


def _sdpa_rows(qrows, keys, vals):
    """torch float64 scaled_dot_product_attention of [B, R, H, d] query rows over
    [B, S, H, d] keys/values, back in [B, R, H, d]."""
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).permute(0, 2, 1, 3)
    return torch.nn.functional.scaled_dot_product_attention(
        t(qrows), t(keys), t(vals)).permute(0, 2, 1, 3).numpy()


def test_joint_layer_is_dense_attention_when_windows_cover_the_clip():
    """Project page, attention-map paragraph, and the H3 key facts (text and audio
    interactions stay dense softmax): with F <= 2c every video window covers the
    clip, so the softmax part of the joint layer is the original dense attention
    of the whole sequence [text; video; audio] for every query row. Compared with
    torch's SDPA over the concatenated sequence."""
    rng = np.random.default_rng(40)
    B, F, N, T, A, H, d, c = 2, 5, 4, 3, 2, 2, 8, 3
    q, k, v, kt, vt, beta, bt, gs, gl = _rand_inputs(rng, B, F, N, T, H, d)
    qt, qa, ka, va = _rand_context(rng, B, T, A, H, d)
    res = O.joint_attention(q, k, v, kt, vt, beta, bt, gs, gl, F, N, c,
                            q_text=qt, q_audio=qa, k_audio=ka, v_audio=va)
    seq_q = np.concatenate([qt, q, qa], 1)
    seq_k = np.concatenate([kt, k, ka], 1)
    seq_v = np.concatenate([vt, v, va], 1)
    dense = _sdpa_rows(seq_q, seq_k, seq_v)
    L = F * N
    np.testing.assert_allclose(res["o_text"], dense[:, :T], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(res["o_soft"], dense[:, T:T + L], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(res["o_audio"], dense[:, T + L:], rtol=1e-12, atol=1e-12)


def test_context_rows_are_dense_for_any_window():
    """Text and audio query rows see every key however small the video window:
    at F = 13, c = 2 they still equal dense SDPA over all video, text and audio
    keys, and their normaliser is the full logsumexp."""
    rng = np.random.default_rng(41)
    B, F, N, T, A, H, d, c = 1, 13, 3, 4, 3, 2, 8, 2
    q, k, v, kt, vt, *_ = _rand_inputs(rng, B, F, N, T, H, d)
    qt, qa, ka, va = _rand_context(rng, B, T, A, H, d)
    keys = np.concatenate([k, kt, ka], 1)
    vals = np.concatenate([v, vt, va], 1)
    for qr in (qt, qa):
        got, lse = O.context_rows(qr, k, v, kt, vt, ka, va, return_lse=True)
        np.testing.assert_allclose(got, _sdpa_rows(qr, keys, vals), rtol=1e-12, atol=1e-12)
        tq = torch.from_numpy(qr).permute(0, 2, 1, 3)
        tk = torch.from_numpy(keys).permute(0, 2, 1, 3)
        ref_lse = torch.logsumexp(tq @ tk.transpose(-1, -2) / np.sqrt(d), -1).permute(0, 2, 1)
        np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=1e-12, atol=1e-12)


def test_audio_keys_reach_every_video_query_and_no_state():
    """An audio key aligned with every query and of large norm takes the whole
    softmax mass of every video row, boundary or not (audio is globally visible);
    the linear branch ignores audio entirely (only the text prompt is written
    into the VDA states)."""
    rng = np.random.default_rng(42)
    B, F, N, T, A, H, d, c = 1, 14, 2, 2, 2, 1, 4, 2
    q, k, v, kt, vt, beta, bt, gs, gl = _rand_inputs(rng, B, F, N, T, H, d)
    q[...] = np.abs(q) + 0.5            # every query in the positive orthant
    _, _, ka, va = _rand_context(rng, B, T, A, H, d)
    ka[0, 0, 0] = 200.0 * np.ones(d)     # dominates every video query's scores
    va[0, 0, 0] = np.arange(1.0, d + 1)
    res = O.joint_attention(q, k, v, kt, vt, beta, bt, gs, gl, F, N, c, k_audio=ka, v_audio=va)
    np.testing.assert_allclose(res["o_soft"][0, :, 0], np.tile(va[0, 0, 0], (F * N, 1)), atol=1e-12)
    no_audio = O.joint_attention(q, k, v, kt, vt, beta, bt, gs, gl, F, N, c)
    np.testing.assert_array_equal(res["o_lin"], no_audio["o_lin"])
    # without audio the video rows reduce to the plain hybrid
    np.testing.assert_array_equal(no_audio["out"], O.hybrid(q, k, v, kt, vt, beta, bt, gs, gl, F, N, c)["out"])
