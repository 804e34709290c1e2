"""GPU parity: every kernel of libolmo3, called through the C ABI, against the
fp64 oracle on the same seeded inputs.

Bars: masks, layer types, cache slots and cache contents bit-exact; QK-norm +
RoPE within bf16 rounding (|err| <= 2^-8 |ref| + 1e-4); attention outputs
max-abs <= 2e-2 and mean-abs <= 2e-3.  LSE: every attention kernel adds the
f32 softmax weights (only the copy of P that feeds the bf16 product is rounded),
so the log-sum-exp carries f32 and ex2.approx rounding only (relative ~1e-6 on
sums of up to 65,536 terms, a few 1e-6 absolute); the bar is 1e-3.
"""
import math

import numpy as np
import pytest
import torch

import oracle.olmo3_oracle as O
from conftest import read_golden
from hybrid_sliding_window_olmo3_b200 import olmo3 as L
from hybrid_sliding_window_olmo3_b200 import workloads as WL

pytestmark = pytest.mark.gpu

TYP = {L.SLIDING: O.SLIDING, L.FULL: O.FULL}
MAX_ABS, MEAN_ABS, LSE_ABS = 2e-2, 2e-3, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L.lib()
    yield
    torch.cuda.synchronize()


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16(a: np.ndarray, dev="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev).to(torch.bfloat16)


def close_attn(got, ref, what=""):
    err = np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64))
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, f"{what}: max {err.max():.3e} mean {err.mean():.3e}"


def close_qk(got, ref, what=""):
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-4
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} elements beyond bf16 rounding, worst {err.max():.3e}"


def new_err():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


# ---------------------------------------------------------------------------
# masks
# ---------------------------------------------------------------------------
def test_mask_table_T5_window2_bit_exact():
    want = np.array([[int(x) for x in r] for r in read_golden("mask_T5_window2.txt")], dtype=np.uint8)
    got = L.attn_mask(5, 2, L.SLIDING).cpu().numpy()
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("T,W,typ", [(1, 1, L.SLIDING), (37, 5, L.SLIDING), (300, 128, L.SLIDING),
                                     (300, 128, L.FULL), (1000, 4096, L.SLIDING), (513, 1, L.SLIDING)])
def test_mask_bit_exact_vs_oracle(T, W, typ):
    got = L.attn_mask(T, W, typ).cpu().numpy().astype(bool)
    want = O.causal_mask(T) if typ == L.FULL else O.sliding_window_mask(T, W)
    np.testing.assert_array_equal(got, want)


# ---------------------------------------------------------------------------
# K1: QK-norm + RoPE
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("B,T,H,G,d,dt,offs", [
    (1, 24, 2, 1, 64, "f32", [0]),
    (2, 5, 32, 32, 128, "bf16", [0, 65530]),
    (2, 3, 40, 8, 128, "bf16", [7, 131072]),
    (1, 130, 4, 2, 128, "bf16", [1000]),
    (3, 2, 2, 2, 64, "f32", [0, 4095, 4096]),
])
def test_qknorm_rope_parity(B, T, H, G, d, dt, offs):
    rng = np.random.default_rng(100 + B * T + H)
    q = rng.standard_normal((B, T, H, d)) * 3
    k = rng.standard_normal((B, T, G, d)) * 3
    v = rng.standard_normal((B, T, G, d))
    gq, gk = rng.uniform(0.5, 1.5, H * d), rng.uniform(0.5, 1.5, G * d)
    if dt == "bf16":
        tq, tk, tv = bf16(q), bf16(k), bf16(v)
    else:
        tq, tk, tv = (torch.from_numpy(x.astype(np.float32)).cuda() for x in (q, k, v))
    q, k, v = f64(tq), f64(tk), f64(tv)   # exact values the GPU sees
    tgq = torch.from_numpy(gq.astype(np.float32)).cuda()
    tgk = torch.from_numpy(gk.astype(np.float32)).cuda()
    gq, gk = f64(tgq), f64(tgk)
    pos = torch.tensor(offs, dtype=torch.int32, device="cuda")
    qh, kh, vo = L.qknorm_rope(tq, tk, tgq, tgk, pos, 1e-6, 5e5, v=tv)
    positions = np.array(offs)[:, None] + np.arange(T)[None, :]
    rq, rk = O.qk_norm_rope(q, k, gq, gk, positions, 1e-6, 5e5)
    close_qk(f64(qh), rq, "q_hat")
    close_qk(f64(kh), rk, "k_hat")
    # v is only cast to bf16 (round to nearest even), bit for bit
    assert torch.equal(vo.cpu(), tv.cpu().to(torch.bfloat16))


@pytest.mark.parametrize("factor,offs", [(8.0, [0, 8191, 65535]), (4.0, [100, 30000, 7]), (1.0, [5, 60000, 1])])
def test_qknorm_rope_yarn_parity(factor, offs):
    rng = np.random.default_rng(150)
    B, T, H, G, d = 3, 4, 32, 32, 128
    tq, tk = bf16(rng.standard_normal((B, T, H, d)) * 2), bf16(rng.standard_normal((B, T, G, d)) * 2)
    gq = torch.rand(H * d, device="cuda") + 0.5
    gk = torch.rand(G * d, device="cuda") + 0.5
    pos = torch.tensor(offs, dtype=torch.int32, device="cuda")
    qh, kh, _ = L.qknorm_rope_yarn(tq, tk, gq, gk, pos, factor=factor, original_context=8192)
    inv = O.yarn_inv_freq(d, 5e5, factor, 8192, 32.0, 1.0)
    positions = np.array(offs)[:, None] + np.arange(T)[None, :]
    rq, rk = O.qk_norm_rope_with(f64(tq), f64(tk), f64(gq), f64(gk), positions, inv, O.yarn_mscale(factor))
    close_qk(f64(qh), rq, "yarn q_hat")
    close_qk(f64(kh), rk, "yarn k_hat")
    if factor == 1.0:  # the same table as plain RoPE: bit for bit
        pq, pk, _ = L.qknorm_rope(tq, tk, gq, gk, pos)
        assert torch.equal(pq, qh) and torch.equal(pk, kh)


def test_qknorm_rope_in_place():
    rng = np.random.default_rng(7)
    B, T, H, G, d = 2, 9, 8, 4, 128
    tq, tk = bf16(rng.standard_normal((B, T, H, d))), bf16(rng.standard_normal((B, T, G, d)))
    q0, k0 = f64(tq), f64(tk)
    gq = torch.rand(H * d, device="cuda") + 0.5
    gk = torch.rand(G * d, device="cuda") + 0.5
    pos = torch.tensor([3, 40000], dtype=torch.int32, device="cuda")
    L.qknorm_rope(tq, tk, gq, gk, pos, q_out=tq, k_out=tk)
    rq, rk = O.qk_norm_rope(q0, k0, f64(gq), f64(gk), np.array([3, 40000])[:, None] + np.arange(T))
    close_qk(f64(tq), rq, "in-place q")
    close_qk(f64(tk), rk, "in-place k")


# ---------------------------------------------------------------------------
# K2: KV append (bit-exact slots and contents; canary rows around the cache)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("typ,W,cap,B,T,offs", [
    (L.SLIDING, 4, 4, 1, 16, [0]),
    (L.SLIDING, 4, 4, 2, 1, [16, 3]),
    (L.SLIDING, 64, 64, 3, 50, [0, 30, 100]),
    (L.SLIDING, 64, 64, 2, 200, [5, 0]),
    (L.FULL, 4096, 200, 2, 17, [0, 150]),
    (L.FULL, 4096, 64, 1, 64, [0]),
])
def test_kv_append_bit_exact(typ, W, cap, B, T, offs):
    G, d, pad = 2, 128, 3
    rng = np.random.default_rng(200 + T)
    kn, vn = bf16(rng.standard_normal((B, T, G, d))), bf16(rng.standard_normal((B, T, G, d)))
    total = B * cap + 2 * pad
    sentinel = 4096.0  # exactly representable in bf16
    ck = torch.full((total, G, d), sentinel, dtype=torch.bfloat16, device="cuda")
    cv = torch.full((total, G, d), -sentinel, dtype=torch.bfloat16, device="cuda")
    base = torch.tensor([pad + b * cap for b in range(B)], dtype=torch.int64, device="cuda")
    cache = L.KVCache(typ, B, G, d, W, capacity=cap, k=ck, v=cv, seq_base=base)
    slot_out = torch.empty((B, T), dtype=torch.int32, device="cuda")
    err = new_err()
    L.kv_append(cache, kn, vn, torch.tensor(offs, dtype=torch.int32, device="cuda"), slot_out, err)
    want_slots = O.append_slots(offs, T, TYP[typ], cap)
    np.testing.assert_array_equal(slot_out.cpu().numpy(), want_slots)
    assert err.item() == 0
    # expected cache: the oracle's replay of every row in order
    exp_k = np.full((total, G, d), sentinel)
    exp_v = np.full((total, G, d), -sentinel)
    kn64, vn64 = f64(kn), f64(vn)
    for b in range(B):
        oc = O.KVCache(TYP[typ], cap, G, d)
        oc.append(range(offs[b], offs[b] + T), kn64[b], vn64[b])
        for s in range(cap):
            if oc.pos[s] >= 0:
                exp_k[pad + b * cap + s] = oc.k[s]
                exp_v[pad + b * cap + s] = oc.v[s]
    np.testing.assert_array_equal(f64(ck), exp_k)
    np.testing.assert_array_equal(f64(cv), exp_v)


def test_kv_append_capacity_error_skips_rows():
    B, T, G, d, cap = 1, 6, 1, 64, 8
    kn = bf16(np.ones((B, T, G, d)))
    ck = torch.zeros((cap, G, d), dtype=torch.bfloat16, device="cuda")
    cv = torch.zeros_like(ck)
    cache = L.KVCache(L.FULL, B, G, d, 4096, capacity=cap, k=ck, v=cv)
    slot_out = torch.empty((B, T), dtype=torch.int32, device="cuda")
    err = new_err()
    L.kv_append(cache, kn, kn, torch.tensor([5], dtype=torch.int32, device="cuda"), slot_out, err)
    assert slot_out.cpu().tolist() == [[5, 6, 7, -1, -1, -1]]
    assert err.item() & L.DEVERR_CAPACITY
    assert f64(ck)[5:].min() == 1.0 and f64(ck)[:5].max() == 0.0


# ---------------------------------------------------------------------------
# K3: prefill attention (tcgen05)
# ---------------------------------------------------------------------------
PREFILL_CASES = [
    # B, T, H, G, d, type, window, q scale
    (1, 16, 2, 1, 64, L.SLIDING, 4, 1.0),
    (1, 16, 2, 1, 64, L.FULL, 4, 1.0),
    (1, 300, 4, 2, 128, L.SLIDING, 200, 1.0),
    (2, 257, 5, 1, 128, L.SLIDING, 128, 1.0),
    (1, 384, 2, 2, 64, L.FULL, 4096, 1.0),
    (1, 255, 2, 2, 128, L.SLIDING, 256, 1.0),
    (1, 256, 2, 2, 128, L.SLIDING, 256, 1.0),
    (1, 257, 2, 2, 128, L.SLIDING, 256, 1.0),
    (1, 1, 1, 1, 128, L.SLIDING, 4096, 1.0),
    (1, 700, 2, 1, 128, L.SLIDING, 1, 1.0),
    (1, 640, 10, 2, 128, L.SLIDING, 129, 1.0),
    (3, 1000, 2, 2, 128, L.FULL, 4096, 1.0),
    (1, 777, 4, 4, 128, L.SLIDING, 300, 4.0),   # peaky logits: exercises the O rescale
    (1, 520, 2, 1, 64, L.FULL, 4096, 6.0),
]


@pytest.mark.parametrize("B,T,H,G,d,typ,W,qs", PREFILL_CASES)
def test_prefill_parity(B, T, H, G, d, typ, W, qs):
    rng = np.random.default_rng(300 + T + H + d)
    tq = bf16(rng.standard_normal((B, T, H, d)) * qs)
    tk = bf16(rng.standard_normal((B, T, G, d)))
    tv = bf16(rng.standard_normal((B, T, G, d)))
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    err = new_err()
    out = L.attn_prefill(tq, tk, tv, typ, W, lse=lse, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ro, rl = O.prefill_attention(f64(tq), f64(tk), f64(tv), TYP[typ], W)
    close_attn(f64(out), ro, "prefill out")
    assert np.abs(lse.cpu().numpy() - rl).max() <= LSE_ABS


def _sampled_prefill(B, T, H, G, d, seed, rows):
    for typ in (L.SLIDING, L.FULL):
        q, k, v, _, _ = WL.qkv_bf16(B, T, H, G, d, seed, layer=typ)
        tq, tk, tv = q.cuda(), k.cuda(), v.cuda()
        out = L.attn_prefill(tq, tk, tv, typ, 4096)
        torch.cuda.synchronize()
        got = f64(out[:, rows])
        ro, _ = O.prefill_attention(f64(q), f64(k), f64(v), TYP[typ], 4096, rows=rows)
        close_attn(got, ro, f"sampled prefill type {typ}")


def test_prefill_7b_full_size_sampled_rows():
    rng = np.random.default_rng(1)
    rows = sorted(set([0, 1, 127, 128, 129, 4094, 4095, 4096, 4097, 6000, 8190, 8191] +
                      rng.integers(0, 8192, 8).tolist()))
    _sampled_prefill(1, 8192, 32, 32, 128, WL.WORKLOADS["7b-prefill"].seed, rows)


def test_prefill_32b_full_size_sampled_rows():
    rng = np.random.default_rng(2)
    rows = sorted(set([0, 255, 4095, 4096, 8191] + rng.integers(0, 8192, 5).tolist()))
    _sampled_prefill(2, 8192, 40, 8, 128, WL.WORKLOADS["32b-prefill"].seed, rows)


# ---------------------------------------------------------------------------
# K4: decode attention over ring / linear caches
# ---------------------------------------------------------------------------
def _decode_case(B, H, G, d, typ, W, lens, seed, num_splits=0, q_scale=1.0):
    rng = np.random.default_rng(seed)
    cap = W if typ == L.SLIDING else max(lens) + 5
    ocs, base = [], []
    ck = torch.zeros((B * cap, G, d), dtype=torch.bfloat16, device="cuda")
    cv = torch.zeros_like(ck)
    for b, n in enumerate(lens):
        oc = O.KVCache(TYP[typ], cap, G, d)
        first = max(0, n - cap) if typ == L.SLIDING else 0   # earlier rows are overwritten anyway
        rows_k = f64(bf16(rng.standard_normal((n - first, G, d)), "cpu"))
        rows_v = f64(bf16(rng.standard_normal((n - first, G, d)), "cpu"))
        oc.append(range(first, n), rows_k, rows_v)
        valid = oc.valid()
        ck[b * cap:(b + 1) * cap][torch.from_numpy(valid).cuda()] = bf16(oc.k[valid])
        cv[b * cap:(b + 1) * cap][torch.from_numpy(valid).cuda()] = bf16(oc.v[valid])
        ocs.append(oc)
    cache = L.KVCache(typ, B, G, d, W, capacity=cap, k=ck, v=cv)
    tq = bf16(rng.standard_normal((B, H, d)) * q_scale)
    kv_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    err = new_err()
    out = L.attn_decode(tq, cache, kv_len, max(lens), lse=lse, err=err, num_splits=num_splits)
    torch.cuda.synchronize()
    assert err.item() == 0
    ro, rl = O.decode_attention(f64(tq), ocs, [n - 1 for n in lens], TYP[typ], W)
    close_attn(f64(out), ro, "decode out")
    assert np.abs(lse.cpu().numpy() - rl).max() <= LSE_ABS


@pytest.mark.parametrize("typ", [L.SLIDING, L.FULL])
@pytest.mark.parametrize("B,H,G,d,W,lens", [
    (6, 2, 1, 64, 4, [1, 3, 4, 5, 8, 9]),
    (5, 4, 2, 128, 256, [255, 256, 257, 512, 513]),
    (3, 10, 2, 128, 4096, [1000, 33, 4097]),
    (2, 8, 1, 128, 64, [100, 64]),
    (4, 6, 2, 64, 128, [1, 2, 127, 300]),
    (2, 32, 2, 128, 4096, [70000, 4100]),        # 16 query heads per key/value head
    (3, 40, 8, 128, 4096, [65537, 64, 65]),      # 32B shapes across a 64-key tile edge
])
def test_decode_parity(typ, B, H, G, d, W, lens):
    _decode_case(B, H, G, d, typ, W, lens, seed=400 + sum(lens))


@pytest.mark.parametrize("splits", [1, 3, 7, 200])
@pytest.mark.parametrize("H,G", [(4, 4), (10, 2)])
def test_decode_split_count_does_not_change_the_result(splits, H, G):
    _decode_case(3, H, G, 128, L.FULL, 4096, [5000, 1, 777], seed=9, num_splits=splits, q_scale=3.0)


def test_decode_bad_kv_len_sets_error_and_zeroes_only_that_sequence():
    B, H, G, d, cap = 3, 2, 2, 128, 64
    ck = bf16(np.random.default_rng(3).standard_normal((B * cap, G, d)))
    cache = L.KVCache(L.FULL, B, G, d, 4096, capacity=cap, k=ck, v=ck.clone())
    q = bf16(np.random.default_rng(4).standard_normal((B, H, d)))
    err = new_err()
    out = L.attn_decode(q, cache, torch.tensor([10, 0, 65], dtype=torch.int32, device="cuda"), 65, err=err)
    torch.cuda.synchronize()
    assert err.item() & L.DEVERR_KV_LEN
    o = f64(out)
    assert np.all(o[1] == 0) and np.all(o[2] == 0) and np.abs(o[0]).sum() > 0


def _sampled_decode(B, H, G, d, lens, seed, check):
    """Random caches on the device; the oracle recomputes the sequences in `check`."""
    for typ in (L.SLIDING, L.FULL):
        cap = 4096 if typ == L.SLIDING else int(max(lens))
        n_slots = B * cap
        ck = WL.randn_bf16((n_slots, G, d), seed * 10 + typ, "cuda")
        cv = WL.randn_bf16((n_slots, G, d), seed * 10 + typ + 5, "cuda")
        cache = L.KVCache(typ, B, G, d, 4096, capacity=cap, k=ck, v=cv)
        q = WL.randn_bf16((B, H, d), seed + 77, "cuda")
        kv_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
        err = new_err()
        out = L.attn_decode(q, cache, kv_len, int(max(lens)), err=err)
        torch.cuda.synchronize()
        assert err.item() == 0
        for b in check:
            n = int(lens[b])
            oc = O.KVCache(TYP[typ], cap, G, d)
            first = max(0, n - cap) if typ == L.SLIDING else 0
            slots = [(p % cap if typ == L.SLIDING else p) for p in range(first, n)]
            rows_k = f64(ck[b * cap:(b + 1) * cap])[slots]
            rows_v = f64(cv[b * cap:(b + 1) * cap])[slots]
            oc.append(range(first, n), rows_k, rows_v)
            ro, _ = O.decode_attention(f64(q[b:b + 1]), [oc], [n - 1], TYP[typ], 4096)
            close_attn(f64(out[b:b + 1]), ro, f"decode seq {b} type {typ}")
        del ck, cv, cache
        torch.cuda.empty_cache()


def test_decode_7b_full_size_sampled():
    wl = WL.WORKLOADS["7b-decode"]
    _sampled_decode(32, 32, 32, 128, [wl.context + 1] * 32, wl.seed, check=[0, 31])


def test_decode_32b_full_size_sampled():
    wl = WL.WORKLOADS["32b-decode"]
    _sampled_decode(8, 40, 8, 128, [wl.context + 1] * 8, wl.seed, check=[0, 7])


def test_decode_ragged_7b_full_size_sampled():
    wl = WL.WORKLOADS["ragged-7b-decode"]
    lens = WL.ragged_lengths(64, wl.seed).tolist()
    order = np.argsort(lens)
    _sampled_decode(64, 32, 32, 128, lens, wl.seed, check=[int(order[0]), int(order[-1]), 5])


# ---------------------------------------------------------------------------
# Chunked prefill: a prompt chunk at an offset over a live cache
# ---------------------------------------------------------------------------
def _cache_from_oracle(ocs, typ, B, G, d, W, cap):
    ck = torch.zeros((B * cap, G, d), dtype=torch.bfloat16, device="cuda")
    cv = torch.zeros_like(ck)
    for b, oc in enumerate(ocs):
        valid = torch.from_numpy(oc.valid()).cuda()
        ck[b * cap:(b + 1) * cap][valid] = bf16(oc.k[oc.valid()])
        cv[b * cap:(b + 1) * cap][valid] = bf16(oc.v[oc.valid()])
    return L.KVCache(typ, B, G, d, W, capacity=cap, k=ck, v=cv)


@pytest.mark.parametrize("typ,W,H,G,d,p0s,T", [
    (L.SLIDING, 256, 4, 2, 128, [0, 1, 255], 100),
    (L.SLIDING, 256, 4, 2, 128, [256, 257, 600], 300),
    (L.SLIDING, 128, 10, 2, 128, [130, 5], 1),
    (L.SLIDING, 64, 2, 1, 64, [63, 64, 65], 77),
    (L.SLIDING, 128, 4, 1, 64, [130, 0, 300], 77),   # d = 64 through the ring read in place
    (L.FULL, 4096, 4, 4, 128, [0, 5, 700], 129),
    (L.FULL, 4096, 10, 2, 128, [1000, 1], 300),
    (L.FULL, 4096, 2, 1, 64, [64, 3], 1),
])
def test_prefill_chunk_parity(typ, W, H, G, d, p0s, T):
    rng = np.random.default_rng(500 + T + sum(p0s))
    B = len(p0s)
    cap = W if typ == L.SLIDING else max(p0s) + T + 130
    ocs = []
    for p0 in p0s:
        oc = O.KVCache(TYP[typ], cap, G, d)
        first = max(0, p0 - cap) if typ == L.SLIDING else 0
        if p0 > first:
            oc.append(range(first, p0), f64(bf16(rng.standard_normal((p0 - first, G, d)), "cpu")),
                      f64(bf16(rng.standard_normal((p0 - first, G, d)), "cpu")))
        ocs.append(oc)
    cache = _cache_from_oracle(ocs, typ, B, G, d, W, cap)
    tq = bf16(rng.standard_normal((B, T, H, d)))
    tk, tv = bf16(rng.standard_normal((B, T, G, d))), bf16(rng.standard_normal((B, T, G, d)))
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    err = new_err()
    out = L.attn_prefill_chunk(tq, tk, tv, cache, torch.tensor(p0s, dtype=torch.int32, device="cuda"),
                               lse=lse, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ro, rl = O.chunk_attention(f64(tq), f64(tk), f64(tv), ocs, p0s, TYP[typ], W)
    close_attn(f64(out), ro, "chunk out")
    assert np.abs(lse.cpu().numpy() - rl).max() <= LSE_ABS
    # the cache now holds the chunk too, exactly as the oracle's replay
    kh, vh = f64(tk), f64(tv)
    for b, oc in enumerate(ocs):
        oc.append(range(p0s[b], p0s[b] + T), kh[b], vh[b])
        got_k = f64(cache.k[b * cap:(b + 1) * cap])
        np.testing.assert_array_equal(got_k[oc.valid()], oc.k[oc.valid()])


@pytest.mark.parametrize("typ", [L.SLIDING, L.FULL])
def test_chunked_prefill_equals_one_shot(typ):
    rng = np.random.default_rng(77)
    B, H, G, d, W, Ttot = 2, 4, 2, 128, 256, 1000
    q, k, v = (rng.standard_normal((B, Ttot, n, d)) for n in (H, G, G))
    tq, tk, tv = bf16(q), bf16(k), bf16(v)
    ro, _ = O.prefill_attention(f64(tq), f64(tk), f64(tv), TYP[typ], W)
    cache = L.KVCache(typ, B, G, d, W, capacity=Ttot + 64)
    p0 = 0
    for T in (300, 1, 255, 444):
        pos = torch.full((B,), p0, dtype=torch.int32, device="cuda")
        out = L.attn_prefill_chunk(tq[:, p0:p0 + T].contiguous(), tk[:, p0:p0 + T].contiguous(),
                                   tv[:, p0:p0 + T].contiguous(), cache, pos)
        torch.cuda.synchronize()
        close_attn(f64(out), ro[:, p0:p0 + T], f"chunk at {p0}")
        p0 += T
    assert p0 == Ttot


@pytest.mark.parametrize("B,H,G", [(1, 32, 32), (2, 40, 8)])
def test_chunked_prefill_full_size_sampled_rows(B, H, G):
    """The bench's chunked workloads: T = 8192 in four chunks of 2048 through a window-sized
    ring (sliding) or a linear cache (full), checked on sampled rows of every chunk."""
    rng = np.random.default_rng(3 + B)
    T, d, W, C = 8192, 128, 4096, 2048
    rows = sorted(set([0, 2047, 2048, 2049, 4095, 4096, 6143, 6144, 8191] + rng.integers(0, T, 6).tolist()))
    for typ in (L.SLIDING, L.FULL):
        q, k, v, _, _ = WL.qkv_bf16(B, T, H, G, d, 20261206, layer=typ)
        tq, tk, tv = q.cuda(), k.cuda(), v.cuda()
        cache = L.KVCache(typ, B, G, d, W, capacity=W if typ == L.SLIDING else T)
        out = torch.empty_like(tq)
        err = new_err()
        for p0 in range(0, T, C):
            pos = torch.full((B,), p0, dtype=torch.int32, device="cuda")
            out[:, p0:p0 + C] = L.attn_prefill_chunk(tq[:, p0:p0 + C].contiguous(), tk[:, p0:p0 + C].contiguous(),
                                                     tv[:, p0:p0 + C].contiguous(), cache, pos, err=err)
        torch.cuda.synchronize()
        assert err.item() == 0
        ro, _ = O.prefill_attention(f64(q), f64(k), f64(v), TYP[typ], W, rows=rows)
        close_attn(f64(out[:, rows]), ro, f"chunked full size type {typ}")


# ---------------------------------------------------------------------------
# Output side: projection + reordered post-norm + residual (tcgen05 GEMM)
# ---------------------------------------------------------------------------
def close_h(got, ref, n_ref, what=""):
    """h = x + n is rounded once to bf16 (2^-9 |h|); n comes from an f32 product and
    an f32 norm.  The bar allows 2^-8 of |h| + |n| (twice the rounding, plus room
    for the f32 accumulation over K) and 1e-3 absolute."""
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * (np.abs(ref) + np.abs(n_ref)) + 1e-3
    assert (err <= bound).all(), f"{what}: {(err > bound).sum()} elements beyond the bound, worst {err.max():.3e}"


@pytest.mark.parametrize("M,D,K", [(1, 256, 64), (100, 512, 128), (300, 4096, 4096), (130, 264, 192),
                                   (257, 5120, 5120)])
def test_out_proj_postnorm_residual_parity(M, D, K):
    rng = np.random.default_rng(600 + M + D)
    attn = bf16(rng.standard_normal((M, K)))
    w = bf16(rng.standard_normal((D, K)) / np.sqrt(K))
    x = bf16(rng.standard_normal((M, D)))
    g = torch.from_numpy(rng.uniform(0.5, 1.5, D).astype(np.float32)).cuda()
    err = new_err()
    h = L.out_proj_postnorm_residual(attn, w, g, x, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = O.out_proj_postnorm_residual(f64(x), f64(attn), f64(w), f64(g))
    close_h(f64(h), ref, ref - f64(x), "out_proj")


def test_out_proj_in_place_and_7b_sampled_rows():
    rng = np.random.default_rng(9)
    M, D, K = 8192, 4096, 4096
    attn = WL.randn_bf16((M, K), 31, "cuda")
    w = (WL.randn_bf16((D, K), 32, "cuda").float() / 64.0).to(torch.bfloat16)
    x = WL.randn_bf16((M, D), 33, "cuda")
    x0 = x.clone()
    g = torch.rand(D, device="cuda") + 0.5
    L.out_proj_postnorm_residual(attn, w, g, x, h_out=x)   # in place on the residual stream
    torch.cuda.synchronize()
    rows = sorted(set([0, 1, 127, 128, 4095, 8191] + rng.integers(0, M, 6).tolist()))
    ref = O.out_proj_postnorm_residual(f64(x0[rows]), f64(attn[rows]), f64(w), f64(g))
    close_h(f64(x[rows]), ref, ref - f64(x0[rows]), "out_proj 7B rows")


# ---------------------------------------------------------------------------
# Input side: fused QKV projection + QK-norm + RoPE (persistent tcgen05 GEMM)
# ---------------------------------------------------------------------------
def qkv_inputs(B, T, H, G, d, D, seed):
    rng = np.random.default_rng(seed)
    x = bf16(rng.standard_normal((B, T, D)))
    w = bf16(rng.standard_normal(((H + 2 * G) * d, D)) / np.sqrt(D))
    gq = torch.from_numpy(rng.uniform(0.5, 1.5, H * d).astype(np.float32)).cuda()
    gk = torch.from_numpy(rng.uniform(0.5, 1.5, G * d).astype(np.float32)).cuda()
    return x, w, gq, gk


def check_qkv(got, x, w, gq, gk, offs, H, G, d, rows=None, yarn=None, what=""):
    """q and k within bf16 rounding of the oracle (f32 accumulation adds far less);
    v likewise (one rounding of an f32 sum)."""
    B, T, D = x.shape
    xs, qo, ko, vo = f64(x), f64(got[0]), f64(got[1]), f64(got[2])
    pos = np.asarray(offs)[:, None] + np.arange(T)[None, :]
    kw = {}
    if yarn is not None:
        kw = dict(inv_freq=O.yarn_inv_freq(d, 5e5, yarn, 8192), out_scale=O.yarn_mscale(yarn))
    if rows is not None:  # sampled tokens (b, t)
        bi, ti = np.array([r[0] for r in rows]), np.array([r[1] for r in rows])
        xs, pos = xs[bi, ti][None], pos[bi, ti][None]
        qo, ko, vo = qo[bi, ti][None], ko[bi, ti][None], vo[bi, ti][None]
    rq, rk, rv = O.qkv_projection(xs, f64(w), f64(gq), f64(gk), pos, H, G, d, **kw)
    close_qk(qo, rq, what + " q")
    close_qk(ko, rk, what + " k")
    close_qk(vo, rv, what + " v")


@pytest.mark.parametrize("B,T,H,G,d,D,offs", [
    (1, 1, 2, 2, 128, 64, [0]),              # one row, one K slice, one tile each of q, k, v
    (2, 100, 4, 2, 128, 256, [0, 37]),       # ragged second row block, position offsets
    (3, 77, 8, 4, 64, 192, [5, 0, 1000]),    # d = 64: four heads per tile
    (1, 8192, 4, 2, 128, 128, [0]),          # 256 tiles: several per CTA, both accumulator buffers
    (1, 300, 40, 8, 128, 5120, [4000]),      # 32B shapes (GQA 5:1)
    (1, 256, 32, 32, 128, 4096, [0]),        # 7B shapes (MHA)
])
def test_qkv_proj_qknorm_rope_parity(B, T, H, G, d, D, offs):
    x, w, gq, gk = qkv_inputs(B, T, H, G, d, D, 700 + T + D)
    pos = torch.tensor(offs, dtype=torch.int32, device="cuda")
    err = new_err()
    got = L.qkv_proj_qknorm_rope(x, w, gq, gk, pos, H, G, d, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    check_qkv(got, x, w, gq, gk, offs, H, G, d, what=f"qkv {B}x{T} H{H} G{G} d{d} D{D}")


def test_qkv_proj_yarn_and_workspace_reuse():
    B, T, H, G, d, D = 2, 200, 4, 2, 128, 256
    offs = [60000, 123]
    x, w, gq, gk = qkv_inputs(B, T, H, G, d, D, 41)
    pos = torch.tensor(offs, dtype=torch.int32, device="cuda")
    ws = torch.full((L.qkv_proj_workspace_size(B * T),), 0x7f, dtype=torch.uint8, device="cuda")  # stale bytes
    err = new_err()
    a = L.qkv_proj_qknorm_rope(x, w, gq, gk, pos, H, G, d, factor=8.0, workspace=ws, err=err)
    b = L.qkv_proj_qknorm_rope(x, w, gq, gk, pos, H, G, d, factor=8.0, workspace=ws, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    for u, v in zip(a, b):
        assert torch.equal(u, v)
    check_qkv(a, x, w, gq, gk, offs, H, G, d, yarn=8.0, what="qkv yarn")


def test_qkv_proj_matches_unfused_path():
    """The fused kernel against the GEMM + K1 pipeline it replaces, on the same inputs."""
    B, T, H, G, d, D = 1, 384, 8, 2, 128, 512
    x, w, gq, gk = qkv_inputs(B, T, H, G, d, D, 43)
    pos = torch.tensor([17], dtype=torch.int32, device="cuda")
    q, k, v = L.qkv_proj_qknorm_rope(x, w, gq, gk, pos, H, G, d)
    y = (x.float().reshape(T, D) @ w.float().T).reshape(B, T, -1)
    q2, k2, _ = L.qknorm_rope(y[..., :H * d].reshape(B, T, H, d).contiguous(),
                              y[..., H * d:(H + G) * d].reshape(B, T, G, d).contiguous(), gq, gk, pos)
    torch.cuda.synchronize()
    # both round nearly equal f32 values to bf16 once: at most one bf16 ulp apart (2^-7 relative)
    for a, b, n in [(q, q2, "q"), (k, k2, "k"), (v, y[..., (H + G) * d:].reshape(B, T, G, d), "v")]:
        err = np.abs(f64(a) - f64(b))
        assert (err <= 2.0 ** -7 * np.abs(f64(b)) + 1e-4).all(), f"fused vs unfused {n}: worst {err.max():.3e}"


def test_qkv_proj_full_size_sampled_rows():
    """7B at the prefill size (8192 tokens, D 4096, N 12288) and 32B at 2 x 8192."""
    rng = np.random.default_rng(12)
    for (B, T, H, G, D, seed) in [(1, 8192, 32, 32, 4096, 51), (2, 8192, 40, 8, 5120, 52)]:
        d = 128
        x = WL.randn_bf16((B, T, D), seed, "cuda")
        w = (WL.randn_bf16(((H + 2 * G) * d, D), seed + 1, "cuda").float() / math.sqrt(D)).to(torch.bfloat16)
        gq = torch.rand(H * d, device="cuda") + 0.5
        gk = torch.rand(G * d, device="cuda") + 0.5
        offs = [0] * B
        pos = torch.tensor(offs, dtype=torch.int32, device="cuda")
        err = new_err()
        got = L.qkv_proj_qknorm_rope(x, w, gq, gk, pos, H, G, d, err=err)
        torch.cuda.synchronize()
        assert err.item() == 0
        rows = sorted(set([(0, 0), (0, 127), (0, 128), (B - 1, T - 1)] +
                          [(int(rng.integers(0, B)), int(rng.integers(0, T))) for _ in range(8)]))
        check_qkv(got, x, w, gq, gk, offs, H, G, d, rows=rows, what=f"qkv full-size H{H}")


# ---------------------------------------------------------------------------
# The toy configuration end to end: 6 layers, prefill 16 tokens, 8 decode steps
# ---------------------------------------------------------------------------
def test_toy_pipeline_full_parity():
    wl = WL.WORKLOADS["toy"]
    sh = wl.shape
    T0, steps = wl.T, wl.steps
    layers = WL.toy_layer_inputs(wl.seed, T0 + steps)
    types = L.layer_types(sh.n_layers)
    assert [TYP[t] for t in types] == O.layer_types(sh.n_layers)
    for li, typ in enumerate(types):
        x = layers[li]
        q, k, v = (torch.from_numpy(x[n]).cuda() for n in ("q", "k", "v"))
        gq, gk = torch.from_numpy(x["gain_q"]).cuda(), torch.from_numpy(x["gain_k"]).cuda()
        # oracle over all 24 tokens
        pos_all = np.arange(T0 + steps)[None, :]
        rq, rk = O.qk_norm_rope(x["q"], x["k"], x["gain_q"], x["gain_k"], pos_all, sh.eps, sh.theta)
        rv = x["v"].astype(np.float64)
        # GPU prefill
        zero = torch.zeros(1, dtype=torch.int32, device="cuda")
        qh, kh, vb = L.qknorm_rope(q[:, :T0].contiguous(), k[:, :T0].contiguous(), gq, gk, zero, sh.eps,
                                   sh.theta, v=v[:, :T0].contiguous())
        close_qk(f64(qh), rq[:, :T0], "toy q_hat")
        close_qk(f64(kh), rk[:, :T0], "toy k_hat")
        cache = L.KVCache(typ, 1, sh.G, sh.d, sh.window, capacity=T0 + steps)
        L.kv_append(cache, kh, vb, zero)
        out = L.attn_prefill(qh, kh, vb, typ, sh.window)
        ro, _ = O.prefill_attention(rq[:, :T0], rk[:, :T0], rv[:, :T0], TYP[typ], sh.window)
        close_attn(f64(out), ro, f"toy prefill layer {li}")
        # oracle cache
        oc = O.KVCache(TYP[typ], cache.capacity, sh.G, sh.d)
        oc.append(range(T0), rk[0, :T0], rv[0, :T0])
        for s in range(steps):
            p = T0 + s
            pos = torch.tensor([p], dtype=torch.int32, device="cuda")
            qh1, kh1, vb1 = L.qknorm_rope(q[:, p:p + 1].contiguous(), k[:, p:p + 1].contiguous(), gq, gk, pos,
                                          sh.eps, sh.theta, v=v[:, p:p + 1].contiguous())
            L.kv_append(cache, kh1, vb1, pos)
            o1 = L.attn_decode(qh1[:, 0].contiguous(), cache, torch.tensor([p + 1], dtype=torch.int32,
                                                                          device="cuda"), p + 1)
            oc.append([p], rk[0, p:p + 1], rv[0, p:p + 1])
            ro1, _ = O.decode_attention(rq[:, p], [oc], [p], TYP[typ], sh.window)
            close_attn(f64(o1), ro1, f"toy decode layer {li} step {s}")
            full = O.full_recompute_last_row(rq[:, :p + 1], rk[:, :p + 1], rv[:, :p + 1], TYP[typ], sh.window)
            close_attn(f64(o1), full, f"toy decode vs recompute layer {li} step {s}")
