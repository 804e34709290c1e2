"""olmo3_attn_decode_noalloc: decode for callers that cannot allocate device
memory (a plugin handed only its inputs and outputs, a C caller without an
allocator).  It keeps its split partials in the library's own fixed device
buffer instead of a caller workspace.  Checked through the C ABI against
olmo3_attn_decode (caller workspace) on two calls in a row, so a buffer still
holding the previous call's partials would show up.  Collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from hybrid_sliding_window_olmo3_b200 import olmo3 as L

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def _case(seed, B, H, G, d, typ, W, lens):
    g = torch.Generator(device="cpu").manual_seed(seed)
    cap = W if typ == L.SLIDING else max(lens) + 3
    ck = torch.randn(B * cap, G, d, generator=g).to(torch.bfloat16).cuda()
    cv = torch.randn(B * cap, G, d, generator=g).to(torch.bfloat16).cuda()
    cache = L.KVCache(typ, B, G, d, W, capacity=cap, k=ck, v=cv)
    q = torch.randn(B, H, d, generator=g).to(torch.bfloat16).cuda()
    kv_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    return cache, q, kv_len


def _noalloc(q, cache, kv_len, max_len, out, err, num_splits=0):
    fn = L.lib().olmo3_attn_decode_noalloc
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(L.CacheStruct), ctypes.c_void_p, ctypes.c_int,
                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    s = cache.struct()
    B, H, d = q.shape
    return fn(q.data_ptr(), H, ctypes.byref(s), kv_len.data_ptr(), max_len, out.data_ptr(), None,
              1.0 / np.sqrt(d), num_splits, err.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_decode_matches_workspace_decode_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cases = [  # the second call has other sizes, so stale partials would be read if any were
        (11, 4, 10, 2, 128, L.FULL, 4096, [5000, 17, 4097, 1]),
        (12, 3, 32, 32, 128, L.SLIDING, 4096, [9000, 4095, 300]),
    ]
    for seed, B, H, G, d, typ, W, lens in cases:
        cache, q, kv_len = _case(seed, B, H, G, d, typ, W, lens)
        ref = L.attn_decode(q, cache, kv_len, max(lens))
        out = torch.full_like(q, float("nan"))
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        assert _noalloc(q, cache, kv_len, max(lens), out, err) == L.OK
        torch.cuda.synchronize()
        assert err.item() == 0
        e = (out.float() - ref.float()).abs().cpu().numpy()
        assert np.isfinite(e).all() and e.max() <= MAX_ABS and e.mean() <= MEAN_ABS


def test_noalloc_rejects_requests_beyond_its_buffer():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B, H, G, d = 64, 32, 32, 128
    cache, q, kv_len = _case(13, B, H, G, d, L.FULL, 4096, [8] * B)
    big = 65536
    # the forced split count makes the partials far larger than the built-in buffer
    assert L.attn_decode_workspace_size(B, H, G, d, big, L.FULL, 4096, 2000) > L.NOALLOC_SCRATCH_BYTES
    out = torch.zeros_like(q)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert _noalloc(q, cache, kv_len, big, out, err, num_splits=2000) == L.ERR_WORKSPACE
    torch.cuda.synchronize()
    assert err.item() == 0 and out.abs().sum().item() == 0
