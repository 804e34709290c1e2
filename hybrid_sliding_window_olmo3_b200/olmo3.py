"""Thin ctypes binding of libolmo3 (include/olmo3.h), same names as the C ABI.

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, outputs are allocated with PyTorch when the caller passes none, and
every computation runs in the library's CUDA kernels.  There is no fallback:
if ``libolmo3.so`` is missing, the first call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

SLIDING = 0
FULL = 1
F32 = 0
BF16 = 1

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_WORKSPACE = -3
ERR_CUDA = -4

DEVERR_CAPACITY = 1
DEVERR_KV_LEN = 2
DEVERR_TIMEOUT = 4

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libolmo3.so")

_vp = ctypes.c_void_p
_i = ctypes.c_int
_lib = None


class Olmo3Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status} ({status_string(status)})")


class CacheStruct(ctypes.Structure):
    _fields_ = [("k", _vp), ("v", _vp), ("seq_base", _vp), ("total_slots", ctypes.c_int64),
                ("capacity", _i), ("layer_type", _i), ("window", _i), ("B", _i), ("G", _i), ("d", _i)]


def lib() -> ctypes.CDLL:
    """Loads libolmo3.so (built in-tree by ``hybrid_sliding_window_olmo3_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m hybrid_sliding_window_olmo3_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    L.olmo3_layer_types.argtypes = [_i, ctypes.POINTER(ctypes.c_uint8)]
    L.olmo3_attn_mask.argtypes = [_i, _i, _i, _vp, _vp]
    L.olmo3_qknorm_rope.argtypes = [_vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp,
                                    _i, _i, _i, _i, _i, ctypes.c_float, ctypes.c_double, _vp]
    L.olmo3_kv_append.argtypes = [ctypes.POINTER(CacheStruct), _vp, _vp, _vp, _i, _vp, _vp, _vp]
    L.olmo3_attn_prefill.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                     ctypes.c_float, _vp, _vp, _vp]
    L.olmo3_attn_decode_workspace_size.argtypes = [_i, _i, _i, _i, _i, _i, _i, _i]
    L.olmo3_attn_decode_workspace_size.restype = ctypes.c_size_t
    L.olmo3_attn_decode.argtypes = [_vp, _i, ctypes.POINTER(CacheStruct), _vp, _i, _vp, _vp,
                                    ctypes.c_float, _i, _vp, ctypes.c_size_t, _vp, _vp]
    L.olmo3_status_string.argtypes = [_i]
    L.olmo3_status_string.restype = ctypes.c_char_p
    for name in ("olmo3_layer_types", "olmo3_attn_mask", "olmo3_qknorm_rope", "olmo3_kv_append",
                 "olmo3_attn_prefill", "olmo3_attn_decode"):
        getattr(L, name).restype = _i
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().olmo3_status_string(status).decode()


def _check(fn: str, status: int):
    if status != OK:
        raise Olmo3Error(fn, status)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else _vp(t.data_ptr())


def _stream(stream) -> _vp:
    s = stream if stream is not None else torch.cuda.current_stream()
    return _vp(s.cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


# --------------------------------------------------------------------------
def layer_types(n_layers: int) -> list[int]:
    """0 = sliding, 1 = full for each layer (host only)."""
    buf = (ctypes.c_uint8 * max(n_layers, 1))()
    _check("olmo3_layer_types", lib().olmo3_layer_types(n_layers, buf))
    return [int(buf[i]) for i in range(n_layers)]


def attn_mask(T: int, window: int, layer_type: int, out: Optional[torch.Tensor] = None,
              device=None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((T, T), dtype=torch.uint8, device=device or "cuda")
    _dev(out, "out", torch.uint8, (T, T))
    _check("olmo3_attn_mask", lib().olmo3_attn_mask(T, window, layer_type, _p(out), _stream(stream)))
    return out


def qknorm_rope(q: torch.Tensor, k: torch.Tensor, gain_q: torch.Tensor, gain_k: torch.Tensor,
                pos_offset: torch.Tensor, eps: float = 1e-6, theta: float = 500000.0,
                v: Optional[torch.Tensor] = None, q_out=None, k_out=None, v_out=None, stream=None):
    """Returns (q_hat, k_hat, v_bf16 or None); q [B,T,H,d], k [B,T,G,d] float32 or bfloat16."""
    B, T, H, d = q.shape
    G = k.shape[2]
    if q.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("q must be float32 or bfloat16")
    in_dtype = F32 if q.dtype == torch.float32 else BF16
    _dev(q, "q")
    _dev(k, "k", q.dtype, (B, T, G, d))
    _dev(gain_q, "gain_q", torch.float32, (H * d,))
    _dev(gain_k, "gain_k", torch.float32, (G * d,))
    _dev(pos_offset, "pos_offset", torch.int32, (B,))
    if q_out is None:
        q_out = torch.empty((B, T, H, d), dtype=torch.bfloat16, device=q.device)
    if k_out is None:
        k_out = torch.empty((B, T, G, d), dtype=torch.bfloat16, device=q.device)
    _dev(q_out, "q_out", torch.bfloat16, (B, T, H, d))
    _dev(k_out, "k_out", torch.bfloat16, (B, T, G, d))
    if v is not None:
        _dev(v, "v", q.dtype, (B, T, G, d))
        if v_out is None:
            v_out = torch.empty((B, T, G, d), dtype=torch.bfloat16, device=q.device)
        _dev(v_out, "v_out", torch.bfloat16, (B, T, G, d))
    _check("olmo3_qknorm_rope", lib().olmo3_qknorm_rope(
        _p(q), _p(k), _p(v), in_dtype, _p(gain_q), _p(gain_k), _p(q_out), _p(k_out), _p(v_out),
        _p(pos_offset), B, T, H, G, d, eps, theta, _stream(stream)))
    return q_out, k_out, v_out


class KVCache:
    """A caller-owned per-layer-type cache: K and V bf16 [total_slots, G, d].

    Sliding layers: capacity == window (a ring).  Full layers: capacity = the
    longest context.  Sequence b owns slots seq_base[b] .. seq_base[b] + capacity - 1
    (by default seq_base[b] = b * capacity).
    """

    def __init__(self, layer_type: int, B: int, G: int, d: int, window: int, capacity: Optional[int] = None,
                 device="cuda", k: Optional[torch.Tensor] = None, v: Optional[torch.Tensor] = None,
                 seq_base: Optional[torch.Tensor] = None):
        self.layer_type, self.B, self.G, self.d, self.window = layer_type, B, G, d, window
        self.capacity = window if layer_type == SLIDING else int(capacity)
        if seq_base is None:
            seq_base = torch.arange(B, dtype=torch.int64, device=device) * self.capacity
        self.seq_base = _dev(seq_base, "seq_base", torch.int64, (B,))
        n = B * self.capacity
        self.k = k if k is not None else torch.zeros((n, G, d), dtype=torch.bfloat16, device=device)
        self.v = v if v is not None else torch.zeros((n, G, d), dtype=torch.bfloat16, device=device)
        _dev(self.k, "cache k", torch.bfloat16)
        _dev(self.v, "cache v", torch.bfloat16, tuple(self.k.shape))
        if self.k.shape[1:] != (G, d):
            raise ValueError("cache k must be [total_slots, G, d]")

    def struct(self) -> CacheStruct:
        return CacheStruct(self.k.data_ptr(), self.v.data_ptr(), self.seq_base.data_ptr(), self.k.shape[0],
                           self.capacity, self.layer_type, self.window, self.B, self.G, self.d)


def kv_append(cache: KVCache, k_new: torch.Tensor, v_new: torch.Tensor, pos_offset: torch.Tensor,
              slot_out: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None, stream=None):
    B, T, G, d = k_new.shape
    _dev(k_new, "k_new", torch.bfloat16, (cache.B, T, cache.G, cache.d))
    _dev(v_new, "v_new", torch.bfloat16, (cache.B, T, cache.G, cache.d))
    _dev(pos_offset, "pos_offset", torch.int32, (cache.B,))
    if slot_out is not None:
        _dev(slot_out, "slot_out", torch.int32, (B, T))
    if err is not None:
        _dev(err, "err", torch.int32)
    s = cache.struct()
    _check("olmo3_kv_append", lib().olmo3_kv_append(ctypes.byref(s), _p(k_new), _p(v_new), _p(pos_offset), T,
                                                    _p(slot_out), _p(err), _stream(stream)))
    return slot_out


def attn_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, layer_type: int, window: int,
                 scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None, stream=None):
    B, T, H, d = q.shape
    G = k.shape[2]
    _dev(q, "q", torch.bfloat16)
    _dev(k, "k", torch.bfloat16, (B, T, G, d))
    _dev(v, "v", torch.bfloat16, (B, T, G, d))
    if out is None:
        out = torch.empty_like(q)
    _dev(out, "out", torch.bfloat16, (B, T, H, d))
    if lse is not None:
        _dev(lse, "lse", torch.float32, (B, H, T))
    if err is not None:
        _dev(err, "err", torch.int32)
    sc = 1.0 / math.sqrt(d) if scale is None else scale
    _check("olmo3_attn_prefill", lib().olmo3_attn_prefill(
        _p(q), _p(k), _p(v), _p(out), B, T, H, G, d, layer_type, window, sc, _p(lse), _p(err),
        _stream(stream)))
    return out


def attn_decode_workspace_size(B: int, H: int, G: int, d: int, max_kv_len: int, layer_type: int,
                               window: int, num_splits: int = 0) -> int:
    return int(lib().olmo3_attn_decode_workspace_size(B, H, G, d, max_kv_len, layer_type, window, num_splits))


def attn_decode(q: torch.Tensor, cache: KVCache, kv_len: torch.Tensor, max_kv_len: int,
                scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                lse: Optional[torch.Tensor] = None, num_splits: int = 0,
                workspace: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None, stream=None):
    B, H, d = q.shape
    _dev(q, "q", torch.bfloat16, (cache.B, H, cache.d))
    _dev(kv_len, "kv_len", torch.int32, (cache.B,))
    if out is None:
        out = torch.empty_like(q)
    _dev(out, "out", torch.bfloat16, (B, H, d))
    if lse is not None:
        _dev(lse, "lse", torch.float32, (B, H))
    if err is not None:
        _dev(err, "err", torch.int32)
    need = attn_decode_workspace_size(B, H, cache.G, d, max_kv_len, cache.layer_type, cache.window, num_splits)
    if workspace is None:
        workspace = torch.empty(max(need // 4, 4), dtype=torch.float32, device=q.device)
    _dev(workspace, "workspace")
    sc = 1.0 / math.sqrt(d) if scale is None else scale
    s = cache.struct()
    _check("olmo3_attn_decode", lib().olmo3_attn_decode(
        _p(q), H, ctypes.byref(s), _p(kv_len), max_kv_len, _p(out), _p(lse), sc, num_splits,
        _p(workspace), workspace.numel() * workspace.element_size(), _p(err), _stream(stream)))
    return out


NOALLOC_SCRATCH_BYTES = 16 << 20


def attn_decode_noalloc(q: torch.Tensor, cache: KVCache, kv_len: torch.Tensor, max_kv_len: int,
                        scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                        lse: Optional[torch.Tensor] = None, num_splits: int = 0,
                        err: Optional[torch.Tensor] = None, stream=None):
    """attn_decode without a workspace: the library's own fixed scratch buffer
    (NOALLOC_SCRATCH_BYTES per GPU) holds the split partials.  For callers that
    cannot allocate; concurrent calls on different streams race on the buffer."""
    fn = lib().olmo3_attn_decode_noalloc
    fn.argtypes = [_vp, _i, ctypes.POINTER(CacheStruct), _vp, _i, _vp, _vp, ctypes.c_float, _i, _vp, _vp]
    fn.restype = _i
    B, H, d = q.shape
    _dev(q, "q", torch.bfloat16, (cache.B, H, cache.d))
    _dev(kv_len, "kv_len", torch.int32, (cache.B,))
    if out is None:
        out = torch.empty_like(q)
    _dev(out, "out", torch.bfloat16, (B, H, d))
    if lse is not None:
        _dev(lse, "lse", torch.float32, (B, H))
    if err is not None:
        _dev(err, "err", torch.int32)
    sc = 1.0 / math.sqrt(d) if scale is None else scale
    s = cache.struct()
    _check("olmo3_attn_decode_noalloc", fn(_p(q), H, ctypes.byref(s), _p(kv_len), max_kv_len, _p(out), _p(lse), sc,
                                           num_splits, _p(err), _stream(stream)))
    return out


def attn_prefill_chunk_workspace_size(B: int, T: int, G: int, d: int, layer_type: int, window: int) -> int:
    fn = lib().olmo3_attn_prefill_chunk_workspace_size
    fn.argtypes = [_i, _i, _i, _i, _i, _i]
    fn.restype = ctypes.c_size_t
    return int(fn(B, T, G, d, layer_type, window))


def attn_prefill_chunk(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, cache: KVCache,
                       pos_offset: torch.Tensor, scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                       lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                       err: Optional[torch.Tensor] = None, stream=None):
    """A prompt chunk at positions pos_offset[b] + t attends over its cache and itself; the chunk
    is appended to the cache.  Sliding layers need a workspace (allocated here if not given)."""
    fn = lib().olmo3_attn_prefill_chunk
    fn.argtypes = [_vp, _vp, _vp, ctypes.POINTER(CacheStruct), _vp, _i, _i, _vp, ctypes.c_float, _vp, _vp,
                   ctypes.c_size_t, _vp, _vp]
    fn.restype = _i
    B, T, H, d = q.shape
    _dev(q, "q", torch.bfloat16, (cache.B, T, H, cache.d))
    _dev(k_new, "k_new", torch.bfloat16, (cache.B, T, cache.G, cache.d))
    _dev(v_new, "v_new", torch.bfloat16, (cache.B, T, cache.G, cache.d))
    _dev(pos_offset, "pos_offset", torch.int32, (cache.B,))
    if out is None:
        out = torch.empty_like(q)
    _dev(out, "out", torch.bfloat16, (B, T, H, d))
    if lse is not None:
        _dev(lse, "lse", torch.float32, (B, H, T))
    if err is not None:
        _dev(err, "err", torch.int32)
    need = attn_prefill_chunk_workspace_size(B, T, cache.G, d, cache.layer_type, cache.window)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    sc = 1.0 / math.sqrt(d) if scale is None else scale
    s = cache.struct()
    _check("olmo3_attn_prefill_chunk", fn(_p(q), _p(k_new), _p(v_new), ctypes.byref(s), _p(pos_offset), T, H,
                                          _p(out), sc, _p(lse), _p(workspace), ws_bytes, _p(err), _stream(stream)))
    return out


def qknorm_rope_yarn(q: torch.Tensor, k: torch.Tensor, gain_q: torch.Tensor, gain_k: torch.Tensor,
                     pos_offset: torch.Tensor, eps: float = 1e-6, theta: float = 500000.0, factor: float = 8.0,
                     original_context: int = 8192, beta_fast: float = 32.0, beta_slow: float = 1.0,
                     v: Optional[torch.Tensor] = None, q_out=None, k_out=None, v_out=None, stream=None):
    """qknorm_rope with YaRN-rescaled RoPE (for the full-attention layers of the long-context model)."""
    fn = lib().olmo3_qknorm_rope_yarn
    fn.argtypes = [_vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, ctypes.c_float,
                   ctypes.c_double, ctypes.c_double, _i, ctypes.c_double, ctypes.c_double, _vp]
    fn.restype = _i
    B, T, H, d = q.shape
    G = k.shape[2]
    if q.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("q must be float32 or bfloat16")
    in_dtype = F32 if q.dtype == torch.float32 else BF16
    _dev(q, "q")
    _dev(k, "k", q.dtype, (B, T, G, d))
    _dev(gain_q, "gain_q", torch.float32, (H * d,))
    _dev(gain_k, "gain_k", torch.float32, (G * d,))
    _dev(pos_offset, "pos_offset", torch.int32, (B,))
    q_out = torch.empty((B, T, H, d), dtype=torch.bfloat16, device=q.device) if q_out is None else q_out
    k_out = torch.empty((B, T, G, d), dtype=torch.bfloat16, device=q.device) if k_out is None else k_out
    _dev(q_out, "q_out", torch.bfloat16, (B, T, H, d))
    _dev(k_out, "k_out", torch.bfloat16, (B, T, G, d))
    if v is not None:
        _dev(v, "v", q.dtype, (B, T, G, d))
        v_out = torch.empty((B, T, G, d), dtype=torch.bfloat16, device=q.device) if v_out is None else v_out
        _dev(v_out, "v_out", torch.bfloat16, (B, T, G, d))
    _check("olmo3_qknorm_rope_yarn", fn(_p(q), _p(k), _p(v), in_dtype, _p(gain_q), _p(gain_k), _p(q_out), _p(k_out),
                                        _p(v_out), _p(pos_offset), B, T, H, G, d, eps, theta, factor,
                                        original_context, beta_fast, beta_slow, _stream(stream)))
    return q_out, k_out, v_out


def out_proj_workspace_size(M: int, D: int) -> int:
    fn = lib().olmo3_out_proj_workspace_size
    fn.argtypes = [_i, _i]
    fn.restype = ctypes.c_size_t
    return int(fn(M, D))


def out_proj_postnorm_residual(attn: torch.Tensor, w_o: torch.Tensor, gain: torch.Tensor, x: torch.Tensor,
                               h_out: Optional[torch.Tensor] = None, eps: float = 1e-6,
                               workspace: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None,
                               stream=None):
    """h = x + RMSNorm(attn W_o^T) * gain (output projection + reordered post-norm + residual)."""
    fn = lib().olmo3_out_proj_postnorm_residual
    fn.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, ctypes.c_float, _vp, ctypes.c_size_t, _vp, _vp]
    fn.restype = _i
    M, K = attn.shape
    D = w_o.shape[0]
    _dev(attn, "attn", torch.bfloat16)
    _dev(w_o, "w_o", torch.bfloat16, (D, K))
    _dev(gain, "gain", torch.float32, (D,))
    _dev(x, "x", torch.bfloat16, (M, D))
    if h_out is None:
        h_out = torch.empty_like(x)
    _dev(h_out, "h_out", torch.bfloat16, (M, D))
    if err is not None:
        _dev(err, "err", torch.int32)
    if workspace is None:
        workspace = torch.empty(max(out_proj_workspace_size(M, D), 16), dtype=torch.uint8, device=x.device)
    _check("olmo3_out_proj_postnorm_residual",
           fn(_p(attn), _p(w_o), _p(gain), _p(x), _p(h_out), M, D, K, eps, _p(workspace),
              workspace.numel() * workspace.element_size(), _p(err), _stream(stream)))
    return h_out


def qkv_proj_workspace_size(M: int) -> int:
    fn = lib().olmo3_qkv_proj_workspace_size
    fn.argtypes = [_i]
    fn.restype = ctypes.c_size_t
    return int(fn(M))


def qkv_proj_qknorm_rope(x: torch.Tensor, w_qkv: torch.Tensor, gain_q: torch.Tensor, gain_k: torch.Tensor,
                         pos_offset: torch.Tensor, H: int, G: int, d: int, eps: float = 1e-6,
                         theta: float = 500000.0, factor: float = 1.0, original_context: int = 8192,
                         beta_fast: float = 32.0, beta_slow: float = 1.0, q_out=None, k_out=None, v_out=None,
                         workspace: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None, stream=None):
    """[q | k | v] = x W_qkv^T, then QK-norm + RoPE (YaRN when factor > 1) on q and k, in one kernel."""
    fn = lib().olmo3_qkv_proj_qknorm_rope
    fn.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, ctypes.c_float,
                   ctypes.c_double, ctypes.c_double, _i, ctypes.c_double, ctypes.c_double, _vp, ctypes.c_size_t,
                   _vp, _vp]
    fn.restype = _i
    B, T, D = x.shape
    _dev(x, "x", torch.bfloat16)
    _dev(w_qkv, "w_qkv", torch.bfloat16, ((H + 2 * G) * d, D))
    _dev(gain_q, "gain_q", torch.float32, (H * d,))
    _dev(gain_k, "gain_k", torch.float32, (G * d,))
    _dev(pos_offset, "pos_offset", torch.int32, (B,))
    q_out = torch.empty((B, T, H, d), dtype=torch.bfloat16, device=x.device) if q_out is None else q_out
    k_out = torch.empty((B, T, G, d), dtype=torch.bfloat16, device=x.device) if k_out is None else k_out
    v_out = torch.empty((B, T, G, d), dtype=torch.bfloat16, device=x.device) if v_out is None else v_out
    _dev(q_out, "q_out", torch.bfloat16, (B, T, H, d))
    _dev(k_out, "k_out", torch.bfloat16, (B, T, G, d))
    _dev(v_out, "v_out", torch.bfloat16, (B, T, G, d))
    if err is not None:
        _dev(err, "err", torch.int32)
    if workspace is None:
        workspace = torch.empty(max(qkv_proj_workspace_size(B * T), 16), dtype=torch.uint8, device=x.device)
    _check("olmo3_qkv_proj_qknorm_rope",
           fn(_p(x), _p(w_qkv), _p(gain_q), _p(gain_k), _p(q_out), _p(k_out), _p(v_out), _p(pos_offset), B, T, H, G,
              d, D, eps, theta, factor, original_context, beta_fast, beta_slow, _p(workspace),
              workspace.numel() * workspace.element_size(), _p(err), _stream(stream)))
    return q_out, k_out, v_out
