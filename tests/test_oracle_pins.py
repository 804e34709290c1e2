"""Pins of the fp64 oracle against what the pages and mathematics fix (CPU only).

Each test checks the oracle against something other than itself: a value
printed on a page (fixtures in tests/golden/, each citing its page and
section), a closed form, an invariant, a textbook routine, or a brute force
written independently with pure-Python loops.  The mutation tests at the end
plant plausible mistakes in the oracle and check that some pin catches each.
"""
import math

import numpy as np
import pytest
from scipy.special import softmax as sp_softmax

import oracle.olmo3_oracle as O
from conftest import read_golden


# ----------------------------------------------------------------------------
# check functions: each returns True when the oracle satisfies the pin.  They
# are reused by the mutation tests below.
# ----------------------------------------------------------------------------
def check_mask_table():
    rows = read_golden("mask_T5_window2.txt")
    want = np.array([[int(x) for x in r] for r in rows], dtype=bool)
    return np.array_equal(O.sliding_window_mask(5, 2), want)


def check_layer_type_examples():
    ok = True
    for r in read_golden("layer_types.txt"):
        n = int(r[0])
        ok &= O.layer_types(n) == r[1:]
    return ok


def check_window3_token4():
    ok = True
    for r in read_golden("window3_token4.txt"):
        ty, w, t = r[0], int(r[1]), int(r[2])
        want = [int(x) for x in r[3:]]
        T = t + 1
        m = O.causal_mask(T) if ty == O.FULL else O.sliding_window_mask(T, w)
        ok &= list(np.nonzero(m[t])[0]) == want
        # the same through the position predicate used by attention
        got = [s for s in range(T) if O.allowed(t, s, ty, w)]
        ok &= got == want
    return ok


def check_qknorm_example():
    g = {r[0]: [float(x) for x in r[1:]] for r in read_golden("qknorm_example.txt")}
    x = np.array(g["input"])
    ok = abs(float(x @ x) - g["dot_before"][0]) < 1e-9
    y = O.rms_norm(x, np.ones(2), 1e-6)
    ok &= bool(np.all(np.abs(y - np.array(g["normed"])) <= 0.005))
    ok &= abs(float(y @ y) - g["dot_after"][0]) <= 0.005
    # the same through the full QK-norm + RoPE path at position 0 (RoPE is the identity there)
    qh, kh = O.qk_norm_rope(x.reshape(1, 1, 1, 2), x.reshape(1, 1, 1, 2), np.ones(2),
                            np.ones(2), np.zeros((1, 1)), 1e-6, 5e5)
    ok &= abs(float(qh.ravel() @ kh.ravel()) - g["dot_after"][0]) <= 0.005
    return bool(ok)


def check_rope_slowest_pair():
    ok = True
    for r in read_golden("rope_slowest_pair.txt"):
        theta, rad, turn = float(r[0]), float(r[1]), float(r[2])
        w = O.rope_inv_freq(128, theta)[63]
        digits = len(r[1].split("e")[0].replace(".", ""))  # page precision
        ok &= abs(w - rad) <= 0.5 * 10 ** (math.floor(math.log10(rad)) - digits + 1) + 1e-18
        ok &= abs(2 * math.pi / w - turn) / turn < 0.02
        # rope() really turns pair 63 by that angle per position
        x = np.zeros((1, 128))
        x[0, 63] = 1.0
        for p in (1, 1000):
            y = O.rope(x, p, theta)[0]
            ang = math.atan2(abs(y[127]), y[63])
            ok &= abs(ang - ((p * w) % (2 * math.pi))) < 1e-9
    return bool(ok)


def check_rope_pairing():
    """Rotate-half: pair i is (i, i + d/2); nothing else mixes."""
    d = 16
    ok = True
    for i in range(d):
        x = np.zeros((1, d))
        x[0, i] = 1.0
        y = O.rope(x, 7, 10.0)[0]
        partner = (i + d // 2) % d
        nz = set(np.nonzero(np.abs(y) > 1e-12)[0])
        ok &= nz <= {i, partner} and partner in nz
    return bool(ok)


def check_gqa_equals_repeated_mha(rng=np.random.default_rng(5)):
    B, T, H, G, d = 1, 7, 6, 2, 4
    q = rng.standard_normal((B, T, H, d))
    k = rng.standard_normal((B, T, G, d))
    v = rng.standard_normal((B, T, G, d))
    o1, l1 = O.prefill_attention(q, k, v, O.SLIDING, 3)
    rep = H // G
    o2, l2 = O.prefill_attention(q, np.repeat(k, rep, axis=2), np.repeat(v, rep, axis=2),
                                 O.SLIDING, 3)
    return np.allclose(o1, o2, atol=1e-12) and np.allclose(l1, l2, atol=1e-12)


def brute_attention(q, k, v, typ, window, scale):
    """Independent pure-Python restatement (loops, math.exp) of masked softmax attention."""
    B, T, H, d = q.shape
    G = k.shape[2]
    out = np.zeros_like(q)
    for b in range(B):
        for t in range(T):
            for h in range(H):
                g = (h * G) // H
                logits = []
                for s in range(T):
                    if s <= t and (typ == "full" or t - s < window):
                        logits.append((s, scale * sum(q[b, t, h, i] * k[b, s, g, i] for i in range(d))))
                m = max(l for _, l in logits)
                ws = [(s, math.exp(l - m)) for s, l in logits]
                z = sum(w for _, w in ws)
                for i in range(d):
                    out[b, t, h, i] = sum(w * v[b, s, g, i] for s, w in ws) / z
    return out


def check_attention_bruteforce(rng=np.random.default_rng(11)):
    ok = True
    for (B, T, H, G, d) in [(1, 9, 2, 1, 4), (2, 12, 4, 2, 8), (1, 6, 3, 3, 2)]:
        q = rng.standard_normal((B, T, H, d))
        k = rng.standard_normal((B, T, G, d))
        v = rng.standard_normal((B, T, G, d))
        for typ, w in [("sliding", 1), ("sliding", 3), ("sliding", T), ("full", 2)]:
            sc = 1.0 / math.sqrt(d)
            o, _ = O.prefill_attention(q, k, v, typ, w, sc)
            ok &= np.allclose(o, brute_attention(q, k, v, typ, w, sc), atol=1e-12)
    return bool(ok)


def check_reordered_norm(rng=np.random.default_rng(21)):
    """[CASE] ingredient 6 fixes h = x + RMSNorm(attn W_o^T): the page's example (identity
    W_o), and two consequences of the norm acting on the projected output before the
    residual: h is unchanged when W_o is scaled, and h - x has RMS 1 (unit gains)."""
    g = {r[0]: [float(x) for x in r[1:]] for r in read_golden("reordered_norm_example.txt")}
    attn, x0 = np.array([g["attention_output"]]), np.array([[0.25, -2.0]])
    ok = np.allclose(O.out_proj_postnorm_residual(x0, attn, np.eye(2), np.ones(2)) - x0, [g["added"]], atol=0.005)
    x, a, w = rng.standard_normal((3, 8)), rng.standard_normal((3, 8)), rng.standard_normal((8, 8))
    h1 = O.out_proj_postnorm_residual(x, a, w, np.ones(8), eps=0.0)  # eps 0: the invariances are exact
    ok &= np.allclose(O.out_proj_postnorm_residual(x, a, 7.0 * w, np.ones(8), eps=0.0), h1, atol=1e-12)
    ok &= np.allclose(np.sqrt(np.mean((h1 - x) ** 2, axis=-1)), 1.0, atol=1e-12)
    return bool(ok)


def check_qkv_identity(rng=np.random.default_rng(22)):
    """Identity weights reduce the QKV projection to QK-norm + RoPE of the input's q and k
    slices and hand the v slice through."""
    B, T, H, G, d = 1, 3, 2, 1, 8
    D = (H + 2 * G) * d
    x = rng.standard_normal((B, T, D))
    gq, gk = rng.uniform(0.5, 1.5, H * d), rng.uniform(0.5, 1.5, G * d)
    pos = np.array([[4, 5, 6]])
    qh, kh, v = O.qkv_projection(x, np.eye(D), gq, gk, pos, H, G, d)
    rq, rk = O.qk_norm_rope(x[..., :H * d].reshape(B, T, H, d), x[..., H * d:(H + G) * d].reshape(B, T, G, d),
                            gq, gk, pos)
    return bool(np.allclose(qh, rq, atol=1e-12) and np.allclose(kh, rk, atol=1e-12) and
                np.array_equal(v, x[..., (H + G) * d:].reshape(B, T, G, d)))


def check_chunked_equals_one_shot(rng=np.random.default_rng(23)):
    """A prompt fed in chunks through the cache gives the rows of the one-shot prefill
    ([README] "Inference Pipeline"), for a ring shorter than the prompt too."""
    ok = True
    B, H, G, d, Ttot = 1, 2, 1, 4, 11
    q, k, v = (rng.standard_normal((B, Ttot, n, d)) for n in (H, G, G))
    for typ, W in (("sliding", 3), ("full", 3)):
        ref, _ = O.prefill_attention(q, k, v, typ, W)
        cache = O.KVCache(typ, W if typ == "sliding" else Ttot, G, d)
        p0 = 0
        for T in (4, 1, 6):
            o, _ = O.chunk_attention(q[:, p0:p0 + T], k[:, p0:p0 + T], v[:, p0:p0 + T], [cache], [p0], typ, W)
            ok &= np.allclose(o, ref[:, p0:p0 + T], atol=1e-12)
            cache.append(range(p0, p0 + T), k[0, p0:p0 + T], v[0, p0:p0 + T])
            p0 += T
    return bool(ok)


# ----------------------------------------------------------------------------
# Pins
# ----------------------------------------------------------------------------
def test_mask_table_T5_window2():
    assert check_mask_table()


def test_layer_types_examples():
    assert check_layer_type_examples()


def test_layer_types_counts():
    # 7B: 32 layers with 8 full (3, 7, ..., 31); 32B: 64 layers, 16 full; the 0.30
    # cache ratio of the case study assumes 24 sliding + 8 full of 32.
    t32 = O.layer_types(32)
    assert [i for i, x in enumerate(t32) if x == O.FULL] == list(range(3, 32, 4))
    assert sum(x == O.FULL for x in O.layer_types(64)) == 16
    assert O.layer_types(1) == [O.FULL]


def test_window3_token4():
    assert check_window3_token4()


@pytest.mark.parametrize("T,w", [(5, 2), (9, 1), (17, 4), (33, 32), (10, 10), (8, 100)])
def test_row_count_is_min_t_plus_1_window(T, w):
    m = O.sliding_window_mask(T, w)
    np.testing.assert_array_equal(m.sum(axis=1), np.minimum(np.arange(T) + 1, w))
    np.testing.assert_array_equal(O.allowed_count(T, w), np.minimum(np.arange(T) + 1, w))


@pytest.mark.parametrize("T,w", [(1, 1), (5, 5), (6, 9), (31, 4096)])
def test_window_ge_T_is_ordinary_causal(T, w):
    np.testing.assert_array_equal(O.sliding_window_mask(T, w), np.tril(np.ones((T, T), dtype=bool)))


def test_attention_masks_follow_layer_types():
    ms = O.attention_masks(7, 6, 2)
    for m, ty in zip(ms, O.layer_types(6)):
        if ty == O.FULL:
            np.testing.assert_array_equal(m, np.tril(np.ones((7, 7), dtype=bool)))
        else:
            np.testing.assert_array_equal(m, O.sliding_window_mask(7, 2))


def test_qknorm_example():
    assert check_qknorm_example()


def test_rmsnorm_unit_gain_has_unit_rms():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 4096)) * 7.0
    y = O.rms_norm(x, np.ones(4096), 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-12)
    g = rng.uniform(0.5, 1.5, 4096)
    np.testing.assert_allclose(O.rms_norm(x, g, 1e-6), O.rms_norm(x, np.ones(4096), 1e-6) * g, rtol=1e-12)


def test_qknorm_is_over_the_whole_vector():
    # the page's gain sizes H*d and G*d reproduce the published parameter counts,
    # which fixes the scope of the norm (one gain per feature of the whole vector)
    for r in read_golden("param_counts.txt"):
        V, D, L, H, G, F, tied, total = (int(x) for x in r[1:])
        d = D // H
        gq, gk = H * d, G * d
        q = np.ones((1, 1, H, d))
        k = np.ones((1, 1, G, d))
        qh, kh = O.qk_norm_rope(q, k, np.ones(gq), np.ones(gk), np.zeros((1, 1)))
        assert qh.size == gq and kh.size == gk
        per_layer = D * H * d + 2 * D * G * d + H * d * D + gq + gk + 3 * D * F + 2 * D
        assert (1 if tied else 2) * V * D + L * per_layer + D == total
    # whole-vector scope: per-token RMS over H*d is one, per-head RMS is not
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 3, 4, 8)) * np.array([1, 2, 3, 4])[None, None, :, None]
    qh, _ = O.qk_norm_rope(q, q[:, :, :1], np.ones(32), np.ones(8), np.zeros((1, 3)), 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(qh.reshape(1, 3, 32) ** 2, axis=-1)), 1.0, rtol=1e-12)


def test_rope_slowest_pair():
    assert check_rope_slowest_pair()


def test_rope_pairing_rotate_half():
    assert check_rope_pairing()


def test_rope_preserves_pair_norms_and_is_identity_at_zero():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 3, 128))
    y = O.rope(x, np.array([0, 5, 4096, 65535]), 5e5)
    n0 = x[..., :64] ** 2 + x[..., 64:] ** 2
    n1 = y[..., :64] ** 2 + y[..., 64:] ** 2
    np.testing.assert_allclose(n0, n1, rtol=1e-12)
    np.testing.assert_allclose(y[0], x[0], atol=0)


def test_rope_relative_position_invariance():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 128))
    k = rng.standard_normal((1, 128))
    for (p, s, c) in [(10, 3, 1000), (70000, 65000, 12345), (5, 5, 4096)]:
        a = float(O.rope(q, p, 5e5)[0] @ O.rope(k, s, 5e5)[0])
        b = float(O.rope(q, p + c, 5e5)[0] @ O.rope(k, s + c, 5e5)[0])
        assert abs(a - b) < 1e-9


def test_qknorm_and_rope_commute_with_unit_gains():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((1, 4, 2, 16))
    pos = np.arange(4)[None, :] + 100
    a, _ = O.qk_norm_rope(q, q[:, :, :1], np.ones(32), np.ones(16), pos)
    r = O.rope(q, pos, 5e5)
    b = O.rms_norm(r.reshape(1, 4, 32), np.ones(32)).reshape(q.shape)
    np.testing.assert_allclose(a, b, atol=1e-12)


def test_attention_matches_bruteforce():
    assert check_attention_bruteforce()


def test_attention_window_ge_T_is_textbook_causal_attention():
    rng = np.random.default_rng(7)
    B, T, H, d = 2, 10, 3, 8
    q, k, v = (rng.standard_normal((B, T, H, d)) for _ in range(3))
    o, lse = O.prefill_attention(q, k, v, O.SLIDING, T + 3)
    o_full, _ = O.prefill_attention(q, k, v, O.FULL, 1)
    sc = 1 / math.sqrt(d)
    for b in range(B):
        for h in range(H):
            logits = q[b, :, h] @ k[b, :, h].T * sc
            logits[~np.tril(np.ones((T, T), dtype=bool))] = -np.inf
            ref = sp_softmax(logits, axis=-1) @ v[b, :, h]
            np.testing.assert_allclose(o[b, :, h], ref, atol=1e-12)
            np.testing.assert_allclose(o_full[b, :, h], ref, atol=1e-12)
            np.testing.assert_allclose(lse[b, h], np.log(np.sum(np.exp(logits), axis=-1)), atol=1e-12)


def test_gqa_equals_mha_with_repeated_kv():
    assert check_gqa_equals_repeated_mha()


def _replay(typ, W, cap, ps, G=1, d=4, rng=None):
    c = O.KVCache(typ, cap, G, d)
    ks = rng.standard_normal((len(ps), G, d))
    c.append(ps, ks, ks * 2)
    return c, ks


@pytest.mark.parametrize("W,p", [(4, 0), (4, 3), (4, 4), (4, 9), (5, 23), (1, 6)])
def test_ring_holds_exactly_the_last_window(W, p):
    rng = np.random.default_rng(8)
    c, ks = _replay(O.SLIDING, W, W, list(range(p + 1)), rng=rng)
    held = sorted(int(x) for x in c.pos[c.valid()])
    assert held == list(range(max(0, p - W + 1), p + 1))
    for j in range(W):
        cands = [q for q in range(p + 1) if q % W == j]
        if cands:
            assert c.pos[j] == max(cands)
            np.testing.assert_array_equal(c.k[j], ks[max(cands)])


@pytest.mark.parametrize("typ,cap,p0,T", [("sliding", 4, 0, 16), ("sliding", 4, 6, 3), ("sliding", 5, 3, 5),
                                          ("full", 40, 0, 16), ("full", 40, 17, 1)])
def test_append_slots_match_replay(typ, cap, p0, T):
    slots = O.append_slots([p0], T, typ, cap)[0]
    rng = np.random.default_rng(9)
    c, ks = _replay(typ, cap, cap, list(range(p0, p0 + T)), rng=rng)
    for t, s in enumerate(slots):
        p = p0 + t
        if s >= 0:
            assert c.pos[s] == p and np.array_equal(c.k[s], ks[t])
        else:
            assert p not in set(c.pos.tolist())
    if typ == "sliding":
        assert sum(s >= 0 for s in slots) == min(T, cap)


@pytest.mark.parametrize("typ", ["sliding", "full"])
def test_decode_with_cache_equals_full_recompute(typ):
    rng = np.random.default_rng(10)
    W, H, G, d = 4, 4, 2, 8
    Ttot = 2 * W + 3
    q = rng.standard_normal((1, Ttot, H, d))
    k = rng.standard_normal((1, Ttot, G, d))
    v = rng.standard_normal((1, Ttot, G, d))
    gq, gk = rng.uniform(0.5, 1.5, H * d), rng.uniform(0.5, 1.5, G * d)
    pos = np.arange(Ttot)[None, :]
    qh, kh = O.qk_norm_rope(q, k, gq, gk, pos)
    cap = W if typ == "sliding" else Ttot
    c = O.KVCache(typ, cap, G, d)
    T0 = W - 1  # prefill, then decode across kv_len W-1 .. 2W+3
    c.append(range(T0), kh[0, :T0], v[0, :T0])
    for p in range(T0, Ttot):
        c.append([p], kh[0, p:p + 1], v[0, p:p + 1])
        o, _ = O.decode_attention(qh[:, p], [c], [p], typ, W)
        ref = O.full_recompute_last_row(qh[:, :p + 1], kh[:, :p + 1], v[:, :p + 1], typ, W)
        np.testing.assert_allclose(o, ref, atol=1e-12)


@pytest.mark.parametrize("typ", ["sliding", "full"])
def test_chunked_prefill_equals_one_shot_prefill(typ):
    # "Apply RoPE with position offsets for cache compatibility": feeding a prompt in
    # chunks through the cache must give the rows of the one-shot prefill.
    rng = np.random.default_rng(12)
    W, H, G, d, Ttot = 5, 4, 2, 8, 23
    q = rng.standard_normal((1, Ttot, H, d))
    k = rng.standard_normal((1, Ttot, G, d))
    v = rng.standard_normal((1, Ttot, G, d))
    ref, ref_lse = O.prefill_attention(q, k, v, typ, W)
    cap = W if typ == "sliding" else Ttot
    c = O.KVCache(typ, cap, G, d)
    p0 = 0
    for T in (1, 4, 7, 2, 9):
        o, lse = O.chunk_attention(q[:, p0:p0 + T], k[:, p0:p0 + T], v[:, p0:p0 + T], [c], [p0], typ, W)
        np.testing.assert_allclose(o, ref[:, p0:p0 + T], atol=1e-12)
        np.testing.assert_allclose(lse, ref_lse[:, :, p0:p0 + T], atol=1e-12)
        c.append(range(p0, p0 + T), k[0, p0:p0 + T], v[0, p0:p0 + T])
        p0 += T
    assert p0 == Ttot


def test_yarn_factor_one_is_plain_rope():
    # the only pin the pages allow: YaRN with factor 1 is plain RoPE (no interpolation, no temperature)
    rng = np.random.default_rng(13)
    x = rng.standard_normal((3, 2, 128))
    pos = np.array([0, 77, 65535])
    np.testing.assert_array_equal(O.yarn_inv_freq(128, 5e5, 1.0, 8192), O.rope_inv_freq(128, 5e5))
    assert O.yarn_mscale(1.0) == 1.0
    np.testing.assert_allclose(O.rope_with(x, pos, O.yarn_inv_freq(128, 5e5, 1.0, 8192), O.yarn_mscale(1.0)),
                               O.rope(x, pos, 5e5), atol=1e-12)


def test_yarn_limits_of_the_ramp():
    # the definition's two ends: fast pairs keep their frequency, slow pairs are divided by the factor
    base = O.rope_inv_freq(128, 5e5)
    f = O.yarn_inv_freq(128, 5e5, 8.0, 8192)
    r = 8192 * base / (2 * math.pi)
    np.testing.assert_allclose(f[r >= 32], base[r >= 32], rtol=1e-15)
    np.testing.assert_allclose(f[r <= 1], base[r <= 1] / 8, rtol=1e-15)
    assert np.all(f <= base) and np.all(f >= base / 8)
    assert abs(O.yarn_mscale(8.0) - (1 + 0.1 * math.log(8))) < 1e-15


def test_reordered_norm_example():
    g = {r[0]: [float(x) for x in r[1:]] for r in read_golden("reordered_norm_example.txt")}
    attn = np.array([g["attention_output"]])
    x = np.array([[0.25, -2.0]])
    h = O.out_proj_postnorm_residual(x, attn, np.eye(2), np.ones(2))
    np.testing.assert_allclose(h - x, [g["added"]], atol=0.005)   # the norm acts on the output, before the add
    h3 = O.out_proj_postnorm_residual(x, attn, np.eye(2), np.array([3.0, 0.5]))
    np.testing.assert_allclose(h3 - x, [[3 * 0.8485281, 0.5 * 1.1313708]], atol=1e-6)  # times the gain


def test_out_projection_is_a_plain_matmul():
    # with a gain of zero only the residual survives; with identity weights the projection is the identity
    rng = np.random.default_rng(14)
    x, a = rng.standard_normal((4, 6)), rng.standard_normal((4, 6))
    np.testing.assert_array_equal(O.out_proj_postnorm_residual(x, a, rng.standard_normal((6, 6)), np.zeros(6)), x)
    w = rng.standard_normal((6, 6))
    ref = x + O.rms_norm(np.einsum("mk,nk->mn", a, w), np.ones(6))
    np.testing.assert_allclose(O.out_proj_postnorm_residual(x, a, w, np.ones(6)), ref, atol=1e-12)


def test_qkv_projection_with_identity_weights_is_qknorm_rope_of_the_input():
    rng = np.random.default_rng(15)
    B, T, H, G, d = 2, 3, 4, 2, 8
    D = (H + 2 * G) * d
    x = rng.standard_normal((B, T, D))
    gq, gk = rng.uniform(0.5, 1.5, H * d), rng.uniform(0.5, 1.5, G * d)
    pos = np.array([[0, 1, 2], [40, 41, 42]])
    qh, kh, v = O.qkv_projection(x, np.eye(D), gq, gk, pos, H, G, d)
    rq, rk = O.qk_norm_rope(x[..., :H * d].reshape(B, T, H, d), x[..., H * d:(H + G) * d].reshape(B, T, G, d),
                            gq, gk, pos)
    np.testing.assert_allclose(qh, rq, atol=1e-12)
    np.testing.assert_allclose(kh, rk, atol=1e-12)
    np.testing.assert_allclose(v, x[..., (H + G) * d:].reshape(B, T, G, d), atol=0)


def test_qkv_projection_with_explicit_plain_frequencies_matches_the_default_path():
    rng = np.random.default_rng(16)
    B, T, H, G, d, D = 1, 5, 2, 1, 8, 12
    x, w = rng.standard_normal((B, T, D)), rng.standard_normal(((H + 2 * G) * d, D))
    gq, gk = rng.uniform(0.5, 1.5, H * d), rng.uniform(0.5, 1.5, G * d)
    pos = np.arange(7, 7 + T)[None]
    a = O.qkv_projection(x, w, gq, gk, pos, H, G, d)
    b = O.qkv_projection(x, w, gq, gk, pos, H, G, d, inv_freq=O.rope_inv_freq(d, 500000.0), out_scale=1.0)
    for u, v in zip(a, b):
        np.testing.assert_allclose(u, v, atol=1e-12)
    # a YaRN temperature multiplies the rotated q and k, and leaves v alone
    c = O.qkv_projection(x, w, gq, gk, pos, H, G, d, inv_freq=O.rope_inv_freq(d, 500000.0), out_scale=1.25)
    np.testing.assert_allclose(c[0], 1.25 * a[0], atol=1e-12)
    np.testing.assert_allclose(c[1], 1.25 * a[1], atol=1e-12)
    np.testing.assert_array_equal(c[2], a[2])


def test_kv_sizing_matches_the_pages():
    g = {r[0]: float(r[1]) for r in read_golden("kv_sizing.txt")}
    t32 = O.layer_types(32)
    naive = O.kv_bytes_per_token(32, 32, 128)
    assert naive == g["naive_bytes_per_token"]
    for c in (4096, 8192, 65536, 100000):
        eff = O.kv_cache_bytes(t32, 32, 128, c, 4096)
        assert eff == g["effective_bytes_per_token_const"] * c + g["effective_bytes_per_token_over_c"]
    assert round(naive * 65536 / O.kv_cache_bytes(t32, 32, 128, 65536, 4096), 2) == g["overpay_at_65536"]
    assert round(naive * 8192 / O.kv_cache_bytes(t32, 32, 128, 8192, 4096), 2) == g["overpay_at_8192"]
    ratio = O.kv_cache_bytes(t32, 32, 128, 65536, 4096) / (naive * 65536)
    assert round(ratio, 2) == g["cache_ratio_at_65536"] and ratio == 0.296875


# ----------------------------------------------------------------------------
# Planted mistakes: each mutation of the oracle must make some pin fail.
# ----------------------------------------------------------------------------
def _mut_mask_inclusive(T, window):
    t = np.arange(T)[:, None]
    s = np.arange(T)[None, :]
    return (s <= t) & (t - s <= window)


def _mut_layer_types_no_last(n):
    return [O.FULL if l % 4 == 3 else O.SLIDING for l in range(n)]


def _mut_rms_sum(x, gain, eps=1e-6):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps) * gain


def _mut_inv_freq_i_over_d(d, theta):
    return np.power(float(theta), -np.arange(d // 2) / d)


def _mut_rope_adjacent(x, positions, theta):
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = np.asarray(positions, dtype=np.float64)[..., None, None] * O.rope_inv_freq(d, theta)
    c, s = np.cos(ang), np.sin(ang)
    y = np.empty_like(x)
    y[..., 0::2] = x[..., 0::2] * c - x[..., 1::2] * s
    y[..., 1::2] = x[..., 1::2] * c + x[..., 0::2] * s
    return y


_real_attend = O.attend


def _mut_attend_gqa_modulo(q, q_pos, k, k_pos, v, layer_type, window, scale=None, k_valid=None):
    # kv head h % G instead of h // (H/G)
    H, G = q.shape[2], k.shape[2]
    idx = [h % G for h in range(H)]
    return _real_attend(q, q_pos, np.asarray(k)[:, :, idx], k_pos, np.asarray(v)[:, :, idx],
                        layer_type, window, scale, k_valid)


def _mut_attend_no_scale(q, q_pos, k, k_pos, v, layer_type, window, scale=None, k_valid=None):
    return _real_attend(q, q_pos, k, k_pos, v, layer_type, window, 1.0, k_valid)


def _mut_postnorm_before_projection(x, attn, w_o, gain, eps=1e-6):
    # the norm on the attention output before W_o
    return np.asarray(x, np.float64) + O.rms_norm(np.asarray(attn, np.float64), np.ones(np.shape(attn)[-1]),
                                                   eps) @ np.asarray(w_o, np.float64).T * np.asarray(gain)


def _mut_postnorm_residual_inside(x, attn, w_o, gain, eps=1e-6):
    # the residual added before the norm (pre-norm-like order)
    y = np.asarray(x, np.float64) + np.asarray(attn, np.float64) @ np.asarray(w_o, np.float64).T
    return O.rms_norm(y, gain, eps)


_real_qkv = O.qkv_projection


def _mut_qkv_k_v_swapped(x, w_qkv, gain_q, gain_k, positions, H, G, d, *args, **kw):
    w = np.asarray(w_qkv, np.float64)
    w = np.concatenate([w[:H * d], w[(H + G) * d:], w[H * d:(H + G) * d]])
    return _real_qkv(x, w, gain_q, gain_k, positions, H, G, d, *args, **kw)


def _mut_qkv_prenormed_input(x, w_qkv, gain_q, gain_k, positions, H, G, d, *args, **kw):
    x = np.asarray(x, np.float64)
    return _real_qkv(O.rms_norm(x, np.ones(x.shape[-1])), w_qkv, gain_q, gain_k, positions, H, G, d, *args, **kw)


_real_chunk = O.chunk_attention


def _mut_chunk_ignores_cache(q_hat, k_hat, v, caches, pos_offset, layer_type, window, scale=None):
    empty = [O.KVCache(c.layer_type, c.n_slots, c.k.shape[1], c.k.shape[2]) for c in caches]
    return _real_chunk(q_hat, k_hat, v, empty, pos_offset, layer_type, window, scale)


ALL_CHECKS = [check_mask_table, check_layer_type_examples, check_window3_token4,
              check_qknorm_example, check_rope_slowest_pair, check_rope_pairing,
              check_gqa_equals_repeated_mha, check_attention_bruteforce,
              check_reordered_norm, check_qkv_identity, check_chunked_equals_one_shot]


def test_all_checks_pass_on_the_oracle():
    assert all(c() for c in ALL_CHECKS)


@pytest.mark.parametrize("name,mut", [
    ("sliding_window_mask", _mut_mask_inclusive),
    ("layer_types", _mut_layer_types_no_last),
    ("rms_norm", _mut_rms_sum),
    ("rope_inv_freq", _mut_inv_freq_i_over_d),
    ("rope", _mut_rope_adjacent),
    ("attend", _mut_attend_gqa_modulo),
    ("attend", _mut_attend_no_scale),
    ("out_proj_postnorm_residual", _mut_postnorm_before_projection),
    ("out_proj_postnorm_residual", _mut_postnorm_residual_inside),
    ("qkv_projection", _mut_qkv_k_v_swapped),
    ("qkv_projection", _mut_qkv_prenormed_input),
    ("chunk_attention", _mut_chunk_ignores_cache),
])
def test_planted_mistakes_are_caught(monkeypatch, name, mut):
    monkeypatch.setattr(O, name, mut)
    assert not all(c() for c in ALL_CHECKS), f"no pin caught the mutation of {name}"
