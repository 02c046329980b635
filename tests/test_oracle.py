"""Pins of the CPU oracle against things other than itself (no GPU).

Each test checks the oracle against a value the pages print, a closed form,
an independent formulation (brute force with an explicit mask built from a
literal FIFO simulation, complex-number RoPE) or a library routine (torch's
float64 scaled-dot-product attention, scipy's logsumexp).
"""
from collections import deque

import numpy as np
import pytest
import torch

import golden_io
from oracle import FrameStream, attend, attend_lse, rope2d, visible_frame_ids
from oracle.stream import visible_token_count
from streaming_video_transformer_b200.inputs import small_workload, frame_qkv


# ----------------------------------------------------------------- fixtures
def _two_frame_inputs():
    z = [0.0] * 4
    q = np.array([[[2, 0, 0, 0]], [z], [z]], dtype=np.float64)           # [3,1,4]
    k0 = np.array([[[1, 0, 0, 0]], [z], [z]], dtype=np.float64)
    v0 = np.array([[[1, 0, 0, 0]], [[0, 1, 0, 0]], [[0, 0, 1, 0]]], dtype=np.float64)
    k1 = np.array([[z], [[1, 0, 0, 0]], [z]], dtype=np.float64)
    v1 = np.array([[[0, 0, 0, 1]], [[1, 1, 0, 0]], [z]], dtype=np.float64)
    return q, (k0, v0), (k1, v1)


def test_two_frame_hand_example():
    cases, _ = golden_io.two_frame_cases()
    assert len(cases) == 9
    q, f0, f1 = _two_frame_inputs()
    for S, W, t, row, expected in cases:
        st = FrameStream(patches_per_frame=2, num_special=1, scale_frames=S, sliding_window=W)
        for f in (f0, f1)[:t]:
            st.append_frame(*f)
        k, v = st.visible_kv()
        o = attend(q, k, v)
        np.testing.assert_allclose(o[row, 0], expected, rtol=0, atol=1e-14,
                                   err_msg=f"S={S} W={W} t={t} row={row}")


def test_two_frame_hand_example_without_cross_frame_special():
    cases, _ = golden_io.two_frame_cases(cross_frame_special=False)
    assert len(cases) == 7
    q, f0, f1 = _two_frame_inputs()
    for S, W, t, row, expected in cases:
        st = FrameStream(patches_per_frame=2, num_special=1, scale_frames=S, sliding_window=W,
                         cross_frame_special=False)
        for f in (f0, f1)[:t]:
            st.append_frame(*f)
        k, v = st.visible_kv()
        o = attend(q, k, v)
        np.testing.assert_allclose(o[row, 0], expected, rtol=0, atol=1e-14,
                                   err_msg=f"no retention S={S} W={W} t={t} row={row}")


def test_cache_stats_example_from_pages():
    g = golden_io.kv_file("cache_stats_example.txt")
    st = FrameStream(patches_per_frame=3, num_special=g["num_special"],
                     scale_frames=g["scale_frames"], sliding_window=g["sliding_window"])
    x = np.zeros((g["num_special"] + 3, 1, 4))
    for _ in range(g["frame_count"]):
        st.append_frame(x, x)
    s = st.stats(patch_capacity=g["patch_capacity"])
    for key in ("frame_count", "scale_pages", "live_pages", "free_pages", "special_tokens"):
        assert s[key] == g[key], key


def test_visible_counts_golden():
    vc = golden_io.visible_counts()
    counts = [int(x) for x in vc["tiny"][1]]
    st = FrameStream(16, 6, 2, 4)
    x = np.zeros((22, 1, 4))
    for t in range(1, 13):
        st.append_frame(x, x)
        assert st.num_visible_tokens() == counts[t - 1]
        assert st.visible_kv()[0].shape[0] == counts[t - 1]
    counts_nc = [int(x) for x in vc["tiny_nocross"][1]]
    st_nc = FrameStream(16, 6, 2, 4, cross_frame_special=False)
    for t in range(1, 13):
        st_nc.append_frame(x, x)
        assert st_nc.num_visible_tokens() == counts_nc[t - 1]
        assert st_nc.visible_kv()[0].shape[0] == counts_nc[t - 1]
    # special pages / last page length of the tiny stream at t=12
    body = dict(tok.split("=") for tok in vc["tiny_pages"][1])
    n_sp = 6 * 12
    assert -(-n_sp // 16) == int(body["special_pages"])
    assert n_sp - 16 * (int(body["special_pages"]) - 1) == int(body["last_page_len"])
    # ViT-L steady state: 72 patch pages + 1200 specials after 200 frames
    assert visible_token_count(200, 1369, 6, 8, 64) == int(vc["vitl"][1][0])
    sc, wi, sp = visible_frame_ids(200, 8, 64, False)
    body = dict(tok.split("=") for tok in vc["vitl_pages"][1])
    assert len(sc) + len(wi) == int(body["patch_pages"])


# -------------------------------------------------- brute force with a mask
def _fifo_visibility(events, S, W):
    """Independent literal simulation: a FIFO of live window frames popped
    while it exceeds W after each (non-deferred) append; returns, for the
    final state, the set of frames whose patches are visible and the list
    of surviving frame ids."""
    frames, scale, window = [], [], deque()
    prov = None
    for ev in events:
        if ev[0] == "append":
            fid, deferred = ev[1], ev[2]
            frames.append(fid)
            if len(scale) < S:
                scale.append(fid)
                where = "scale"
            else:
                window.append(fid)
                where = "window"
            prov = (fid, where) if deferred else None
            if not deferred:
                while len(window) > W:
                    window.popleft()
        elif ev[0] == "accept":
            prov = None
            while len(window) > W:
                window.popleft()
        elif ev[0] == "rollback":
            fid, where = prov
            frames.pop()
            (scale if where == "scale" else window).pop()
            prov = None
    return set(scale) | set(window), frames


@pytest.mark.parametrize("cross", [True, False])
@pytest.mark.parametrize("S,W,seed", [(2, 4, 0), (0, 3, 1), (3, 1, 2), (1, 0, 3), (4, 2, 4)])
def test_bruteforce_masked_attention(S, W, seed, cross):
    """Without cross-frame special retention a special token's mask entry is
    its frame's patch visibility; with it, 0 always."""
    rng = np.random.default_rng(seed)
    P, ns, H, D = 5, 2, 2, 8
    st = FrameStream(P, ns, S, W, cross_frame_special=cross)
    all_k, all_v, events, store = {}, {}, [], {}
    fid = 0
    for step in range(11):
        k = rng.standard_normal((ns + P, H, D))
        v = rng.standard_normal((ns + P, H, D))
        deferred = step % 3 == 2
        st.append_frame(k, v, deferred=deferred)
        store[fid] = (k, v)
        events.append(("append", fid, deferred))
        if deferred:
            if rng.random() < 0.5:
                st.rollback_last_frame()
                events.append(("rollback",))
                del store[fid]
            else:
                st.execute_deferred_eviction()
                events.append(("accept",))
        fid += 1
        # brute force: every token of every surviving frame, masked by labels
        vis_patch, frames = _fifo_visibility(events, S, W)
        ks, vs, mask = [], [], []
        for f in frames:
            k_f, v_f = store[f]
            for r in range(ns + P):
                is_special = r < ns
                ks.append(k_f[r]); vs.append(v_f[r])
                visible = (is_special and cross) or f in vis_patch
                mask.append(0.0 if visible else -np.inf)
        K = torch.tensor(np.stack(ks)).permute(1, 0, 2)         # [H,N,D]
        V = torch.tensor(np.stack(vs)).permute(1, 0, 2)
        q = rng.standard_normal((ns + P, H, D))
        Q = torch.tensor(q).permute(1, 0, 2)
        M = torch.tensor(np.array(mask))[None, None, :].expand(H, Q.shape[1], -1)
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=M)
        ref = ref.permute(1, 0, 2).numpy()
        kv_k, kv_v = st.visible_kv()
        o = attend(q, kv_k, kv_v)
        np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


# ------------------------------------------------------------ closed forms
def test_uniform_attention_is_mean_of_visible_v():
    rng = np.random.default_rng(5)
    k = rng.standard_normal((37, 3, 16))
    v = rng.standard_normal((37, 3, 16))
    q = np.zeros((4, 3, 16))
    o, lse = attend_lse(q, k, v)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(0), o.shape), atol=1e-14)
    np.testing.assert_allclose(lse, np.log(37.0), atol=1e-14)


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(6)
    D = 16
    k = rng.standard_normal((50, 1, D)) * 0.01
    v = rng.standard_normal((50, 1, D))
    q = np.zeros((1, 1, D)); q[0, 0, 0] = 1.0
    k[17, 0, :] = 0.0; k[17, 0, 0] = 30.0 * np.sqrt(D)      # score +30 vs ~0
    o = attend(q, k, v)
    np.testing.assert_allclose(o[0, 0], v[17, 0], atol=60 * np.exp(-29.0))


def test_lse_matches_logsumexp_and_sdpa():
    from scipy.special import logsumexp
    rng = np.random.default_rng(7)
    q = rng.standard_normal((9, 2, 32)); k = rng.standard_normal((70, 2, 32))
    v = rng.standard_normal((70, 2, 32))
    o, lse = attend_lse(q, k, v, row_block=4)
    for h in range(2):
        s = q[:, h] @ k[:, h].T / np.sqrt(32)
        np.testing.assert_allclose(lse[:, h], logsumexp(s, axis=1), atol=1e-12)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q).permute(1, 0, 2), torch.tensor(k).permute(1, 0, 2),
        torch.tensor(v).permute(1, 0, 2)).permute(1, 0, 2).numpy()
    np.testing.assert_allclose(o, ref, atol=1e-12)


# --------------------------------------------------------------- invariants
@pytest.mark.parametrize("cross", [True, False])
def test_visible_count_formula_on_random_streams(cross):
    rng = np.random.default_rng(8)
    for _ in range(20):
        P, ns = int(rng.integers(1, 6)), int(rng.integers(0, 4))
        S, W = int(rng.integers(0, 4)), int(rng.integers(0, 5))
        st = FrameStream(P, ns, S, W, cross_frame_special=cross)
        x = np.zeros((ns + P, 1, 4))
        for t in range(1, 15):
            deferred = rng.random() < 0.3
            st.append_frame(x, x, deferred=deferred)
            frames = min(t, S) + min(max(t - S, 0), W + (1 if deferred else 0))
            expect = frames * P + ns * t if cross else frames * (P + ns)
            if ns + P and expect:
                assert st.visible_kv()[0].shape[0] == expect
            if deferred:
                st.rollback_last_frame()
                st.append_frame(x, x)


def test_rollback_restores_outputs_exactly():
    w = small_workload(P=16, ns=6, S=2, W=3, H=2, D=64)
    st = FrameStream(w.P, w.ns, w.S, w.W)
    for t in range(6):
        q, k, v = frame_qkv(w, 0, 0, t)
        st.append_frame(k, v)
    before = attend(q, *st.visible_kv())
    _, k2, v2 = frame_qkv(w, 0, 0, 99)
    st.append_frame(k2, v2, deferred=True)
    during = attend(q, *st.visible_kv())
    assert not np.array_equal(before, during)
    st.rollback_last_frame()
    after = attend(q, *st.visible_kv())
    assert np.array_equal(before, after)


# --------------------------------------------------------------------- RoPE
def _rope_complex(x, ns, grid, theta):
    """Independent form: each (i, i+m/2) pair of a half is one complex number
    multiplied by exp(1j * pos * theta**(-2i/m))."""
    x = np.asarray(x, dtype=np.float64)
    out = x.copy()
    D = x.shape[2]; m = D // 2; half = m // 2
    for p in range(grid * grid):
        for sect, pos in ((0, p // grid), (1, p % grid)):
            base = sect * m
            z = x[ns + p, :, base:base + half] + 1j * x[ns + p, :, base + half:base + m]
            z = z * np.exp(1j * pos * theta ** (-2.0 * np.arange(half) / m))
            out[ns + p, :, base:base + half] = z.real
            out[ns + p, :, base + half:base + m] = z.imag
    return out


def test_rope_against_complex_form_and_identities():
    """The fp32 rotation against the complex form in float64 on the same
    (fp32) inputs: within the fp32 rounding of two products, their
    difference and the tables (3 units of 2^-24 of |a| + |b|)."""
    rng = np.random.default_rng(9)
    ns, grid, theta = 3, 5, 100.0
    x = rng.standard_normal((ns + grid * grid, 2, 16)).astype(np.float32)
    y = rope2d(x, ns, grid, theta)
    assert y.dtype == np.float32
    ref = _rope_complex(x, ns, grid, theta)
    D = x.shape[2]; m = D // 2; half = m // 2
    mag = np.empty_like(ref)
    for base in (0, m):
        pair = np.abs(x[..., base:base + half]) + np.abs(x[..., base + half:base + m])
        mag[..., base:base + half] = pair
        mag[..., base + half:base + m] = pair
    assert np.all(np.abs(y - ref) <= 3.0 * 2.0 ** -24 * mag + 1e-30)
    assert np.max(np.abs(y - ref)) > 0                            # rounding is not hidden
    np.testing.assert_array_equal(y[:ns], x[:ns])                 # specials untouched
    np.testing.assert_array_equal(y[ns], x[ns])                   # patch (0,0): identity, exact
    np.testing.assert_allclose(np.linalg.norm(y.astype(np.float64), axis=2),
                               np.linalg.norm(x.astype(np.float64), axis=2), rtol=1e-6)


def test_rope_unit_vectors_give_fp32_tables_exactly():
    """Rotating the unit vector of feature i returns, exactly, the fp32
    rounding of cos and sin of pos * theta^(-2i/m) (Python's math library,
    float64), with pos the patch's row in the first half and its column in
    the second: rn(1*c) - rn(0*s) = c and rn(1*s) + rn(0*c) = s."""
    import math
    ns, grid, theta, D = 1, 4, 100.0, 16
    m, half = D // 2, D // 4
    for sect in (0, 1):
        for i in range(half):
            x = np.zeros((ns + grid * grid, 1, D), np.float32)
            x[ns:, 0, sect * m + i] = 1.0
            y = rope2d(x, ns, grid, theta)
            for p in range(grid * grid):
                pos = p // grid if sect == 0 else p % grid
                ang = pos * theta ** (-2.0 * i / m)
                assert y[ns + p, 0, sect * m + i] == np.float32(math.cos(ang))
                assert y[ns + p, 0, sect * m + half + i] == np.float32(math.sin(ang))
                others = np.delete(y[ns + p, 0], [sect * m + i, sect * m + half + i])
                assert not np.any(others)


def test_rope_fp32_and_float64_rotations_round_alike_to_bf16():
    """Rounded to bf16, the fp32 rotation and the float64 one agree except
    on elements whose float64 value lies within the fp32 error of a bf16
    rounding boundary: there they differ by one bf16 step, or by the fp32
    error itself where cancellation leaves a value far below |a| + |b|."""
    rng = np.random.default_rng(11)
    ns, grid, theta = 6, 37, 100.0
    x = torch.randn((ns + grid * grid, 4, 64), generator=torch.Generator().manual_seed(11))
    x = x.to(torch.bfloat16).float().numpy()
    a = torch.from_numpy(rope2d(x, ns, grid, theta)).to(torch.bfloat16).double().numpy()
    b = torch.from_numpy(_rope_complex(x, ns, grid, theta)).to(torch.bfloat16).double().numpy()
    diff = a != b
    assert np.mean(diff) < 1e-3
    # one bf16 step of the value, or (after cancellation leaves a tiny value)
    # the fp32 error of the rotation, 3 units of 2^-24 of the pair's |a|+|b|
    D = x.shape[2]; m = D // 2; half = m // 2
    mag = np.empty_like(x, dtype=np.float64)
    for base in (0, m):
        pair = np.abs(x[..., base:base + half]) + np.abs(x[..., base + half:base + m])
        mag[..., base:base + half] = pair
        mag[..., base + half:base + m] = pair
    step = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(b[diff]), 1e-30))) - 7)
    assert np.all(np.abs(a[diff] - b[diff]) <= np.maximum(step * 1.0001, 4 * 2.0 ** -24 * mag[diff]))


def test_rope_dot_product_depends_only_on_offset():
    rng = np.random.default_rng(10)
    ns, grid = 0, 6
    a = rng.standard_normal(16); b = rng.standard_normal(16)
    X = np.tile(a, (grid * grid, 1, 1)); Y = np.tile(b, (grid * grid, 1, 1))
    RX = rope2d(X, ns, grid, 100.0).astype(np.float64)
    RY = rope2d(Y, ns, grid, 100.0).astype(np.float64)
    for (r1, c1, r2, c2) in [(0, 0, 1, 2), (3, 3, 4, 5), (2, 1, 3, 3)]:
        d1 = RX[r1 * grid + c1, 0] @ RY[r2 * grid + c2, 0]
        d2 = RX[(r1 + 1) * grid + c1 - 0, 0] @ RY[(r2 + 1) * grid + c2, 0] if r2 + 1 < grid else d1
        assert abs(d1 - d2) < 1e-5


def test_deferred_frame_visible_set_is_cache_plus_the_frame():
    """Attending a frame without storing it (cache + the frame's own rows)
    sees the same tokens as appending it with eviction deferred: compared
    as sets of rows, with and without special retention."""
    rng = np.random.default_rng(12)
    for cross in (True, False):
        for S, W in ((2, 3), (0, 2), (3, 1), (1, 0)):
            st = FrameStream(3, 2, S, W, cross_frame_special=cross)
            for t in range(7):
                k = rng.standard_normal((5, 1, 4))
                st.append_frame(k, k + 1.0)
                kf = rng.standard_normal((5, 1, 4))
                vf = kf + 1.0
                kc, vc = st.visible_kv()
                plus = np.concatenate([kc, kf])
                st.append_frame(kf, vf, deferred=True)
                kd, _ = st.visible_kv()
                st.rollback_last_frame()
                a = sorted(map(tuple, plus.reshape(len(plus), -1)))
                b = sorted(map(tuple, kd.reshape(len(kd), -1)))
                assert a == b, (cross, S, W, t)
