"""fp64 CPU oracle for OLMo 3 hybrid sliding-window attention (TEST INFRASTRUCTURE).

This module is test infrastructure: only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it.  It is written from the
pages below, in NumPy float64, with no blocking, fusion or reordering beyond the
definitions; it never imports the GPU package.

Sources (page title, section):

* [PATTERN]  "OLMo 3's Sliding-Window Attention Pattern" (scratchllm.com problem
  page): "Which layers are full", "The sliding-window mask" with its
  T = 5 / window = 2 table, "Hint" (row count min(t + 1, window)).
* [CASE]     "Case Study: OLMo 3" (scratchllm.com learn page), "The architecture":
  1. projections / GQA (40 query heads on 8 key/value heads), 2. QK-norm and its
  (30, 40) example, 3. RoPE with theta = 500,000, rotate-half pairing and the
  slowest-pair example, 4. sliding-window attention with the 8-layer and
  window-3 examples and the 0.30 cache ratio.
* [COUNT]    "Count OLMo 3's Parameters" (scratchllm.com problem page), "What to
  count": the QK-norm gains have Hd and Gd features.
* [README]   "Olmo-3 End-to-End Implementation" (GitHub README), "Inference
  Pipeline" (prefill builds the cache, decode one token at a time, RoPE with a
  position offset), "Technical Details" (RMSNorm eps 1e-6; RoPE on q and k only).
* [SERVING]  "Olmo 3 7B" (inference-research record): per-layer-type cache
  management, KV bytes per token and "KV OVERPAY FOR THIS CHECKPOINT".

Readings where the pages leave a step open:

* R1  RMSNorm puts eps inside the square root: x / sqrt(mean(x^2) + eps).
* R2  QK-norm normalises the whole H*d query vector (G*d key vector) of a token.
* R3  QK-norm comes before RoPE (the order of the ingredients in [CASE]).
* R4  RoPE angle a_i = p * theta^(-2i/d), i < d/2, pairs (i, i + d/2):
      x'_i = x_i cos a - x_{i+d/2} sin a,  x'_{i+d/2} = x_{i+d/2} cos a + x_i sin a.
      The direction of rotation is a convention: parity unpinned for the sign
      only (frequencies, pairing, norm preservation and shift invariance are
      pinned by tests).
* R5  Softmax scale defaults to 1/sqrt(d); callers may pass another.
* R6  The cache stores keys after QK-norm and RoPE, at their absolute position.
* R7  Ring slot = p mod window (sliding layers); linear slot = p (full layers).
* R8  GQA: query head h reads key/value head floor(h / (H / G)).
* R13 A prompt chunk at an offset attends over its cache and itself; on a sliding
      layer it attends first and is appended after (appending first would
      overwrite keys its early rows need).
* R14 YaRN on full layers: NTK-by-parts frequencies with the method's ramp bounds
      (beta_fast 32, beta_slow 1) and the temperature 0.1 ln(factor) + 1 on q and
      k.  Parity unpinned beyond factor 1 (factor 1 is plain RoPE, pinned).
* R15 Reordered norm: h = x + RMSNorm(attn W_o^T) over the D model features, one
      gain per feature, eps 1e-6.
* R16 The QKV projection takes the block input as it is (the reordered norm
      leaves it un-normed).
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "SLIDING", "FULL", "layer_types", "sliding_window_mask", "causal_mask",
    "attention_masks", "allowed", "allowed_count", "rms_norm", "rope_inv_freq",
    "rope", "qk_norm_rope", "attend", "prefill_attention", "KVCache",
    "append_slots", "decode_attention", "full_recompute_last_row", "chunk_attention",
    "yarn_inv_freq", "yarn_mscale", "rope_with", "qk_norm_rope_with", "out_proj_postnorm_residual",
    "qkv_projection",
    "kv_bytes_per_token", "kv_cache_bytes",
]

SLIDING = "sliding"
FULL = "full"


# ---------------------------------------------------------------------------
# Layer pattern and masks  ([PATTERN] "Which layers are full",
# "The sliding-window mask"; [CASE] ingredient 4)
# ---------------------------------------------------------------------------
def layer_types(n_layers: int) -> list[str]:
    """Layer l (from 0) is full when l mod 4 == 3 or it is the last layer."""
    last = n_layers - 1
    return [FULL if (l % 4 == 3 or l == last) else SLIDING for l in range(n_layers)]


def sliding_window_mask(T: int, window: int) -> np.ndarray:
    """Boolean (T, T): query t sees key s iff s <= t and t - s < window.

    Built by broadcasting a column of query positions against a row of key
    positions, as the page's hint says (no loop over positions).
    """
    t = np.arange(T)[:, None]
    s = np.arange(T)[None, :]
    return (s <= t) & (t - s < window)


def causal_mask(T: int) -> np.ndarray:
    """The plain causal mask of a full layer: s <= t."""
    t = np.arange(T)[:, None]
    s = np.arange(T)[None, :]
    return s <= t


def attention_masks(T: int, n_layers: int, window: int) -> list[np.ndarray]:
    """One mask per layer following ``layer_types``; full layers get the causal mask."""
    return [causal_mask(T) if ty == FULL else sliding_window_mask(T, window)
            for ty in layer_types(n_layers)]


def allowed(q_pos, k_pos, layer_type: str, window: int) -> np.ndarray:
    """The mask predicate on absolute positions (broadcasting)."""
    q_pos = np.asarray(q_pos)
    k_pos = np.asarray(k_pos)
    ok = k_pos <= q_pos
    if layer_type == SLIDING:
        ok = ok & ((q_pos - k_pos) < window)
    return ok


def allowed_count(T: int, window: int) -> np.ndarray:
    """Allowed keys in each row of the sliding mask: min(t + 1, window)."""
    t = np.arange(T)
    return np.minimum(t + 1, window)


# ---------------------------------------------------------------------------
# QK-norm and RoPE  ([CASE] ingredients 2 and 3; [COUNT] gain sizes;
# [README] "Technical Details")
# ---------------------------------------------------------------------------
def rms_norm(x, gain, eps: float = 1e-6) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * gain over the last axis (reading R1)."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(gain, dtype=np.float64)


def rope_inv_freq(d: int, theta: float) -> np.ndarray:
    """Angle per position of pair i: theta^(-2i/d), i = 0 .. d/2 - 1."""
    i = np.arange(d // 2, dtype=np.float64)
    return np.power(float(theta), -2.0 * i / d)


def rope(x, positions, theta: float) -> np.ndarray:
    """Rotate-half RoPE (reading R4).

    x: [..., n_heads, d]; positions: broadcastable to x.shape[:-2].
    Pair i is (i, i + d/2) inside each head.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    pos = np.asarray(positions, dtype=np.float64)[..., None, None]
    ang = pos * rope_inv_freq(d, theta)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def yarn_inv_freq(d: int, theta: float, factor: float, original_context: int,
                  beta_fast: float = 32.0, beta_slow: float = 1.0) -> np.ndarray:
    """YaRN frequencies (Peng et al., 2023, "NTK-by-parts" interpolation).

    [CASE] ingredient 7 and [SERVING]: RoPE of the full-attention layers is
    rescaled with YaRN, factor 8 from the 8,192 positions of training.  The pages
    give only the factor and the base context; the ramp bounds are the method's
    (beta_fast = 32, beta_slow = 1): parity unpinned beyond factor 1 == plain RoPE.

    Pair i turns r_i = original_context * theta^(-2i/d) / (2 pi) times over the
    original context.  Pairs with r_i >= beta_fast keep their frequency, pairs with
    r_i <= beta_slow are interpolated (frequency / factor), and a linear ramp in r_i
    blends the two in between.
    """
    base = rope_inv_freq(d, theta)
    if factor == 1.0:
        return base
    r = original_context * base / (2.0 * math.pi)
    ramp = np.clip((r - beta_slow) / (beta_fast - beta_slow), 0.0, 1.0)  # 1 = keep, 0 = interpolate
    return base * ramp + (base / factor) * (1.0 - ramp)


def yarn_mscale(factor: float) -> float:
    """YaRN attention temperature: q and k are both scaled by 0.1 ln(factor) + 1
    (so the logits by its square); 1 for factor <= 1."""
    return 1.0 if factor <= 1.0 else 0.1 * math.log(factor) + 1.0


def rope_with(x, positions, inv_freq, out_scale: float = 1.0) -> np.ndarray:
    """Rotate-half RoPE with an explicit frequency per pair, then a scale."""
    x = np.asarray(x, dtype=np.float64)
    half = x.shape[-1] // 2
    ang = np.asarray(positions, dtype=np.float64)[..., None, None] * np.asarray(inv_freq, dtype=np.float64)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1) * out_scale


def qk_norm_rope_with(q, k, gain_q, gain_k, positions, inv_freq, out_scale: float = 1.0,
                      eps: float = 1e-6):
    """QK-norm over the whole vector, then RoPE with the given frequencies and scale."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    B, T, H, d = q.shape
    G = k.shape[2]
    qn = rms_norm(q.reshape(B, T, H * d), gain_q, eps).reshape(B, T, H, d)
    kn = rms_norm(k.reshape(B, T, G * d), gain_k, eps).reshape(B, T, G, d)
    return rope_with(qn, positions, inv_freq, out_scale), rope_with(kn, positions, inv_freq, out_scale)


def qk_norm_rope(q, k, gain_q, gain_k, positions, eps: float = 1e-6,
                 theta: float = 500000.0):
    """QK-norm over the whole H*d / G*d vector, then RoPE at each token's position.

    q: [B, T, H, d], k: [B, T, G, d], gain_q: [H*d], gain_k: [G*d],
    positions: [B, T] absolute positions.  Returns (q_hat, k_hat) in float64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    B, T, H, d = q.shape
    G = k.shape[2]
    qn = rms_norm(q.reshape(B, T, H * d), gain_q, eps).reshape(B, T, H, d)
    kn = rms_norm(k.reshape(B, T, G * d), gain_k, eps).reshape(B, T, G, d)
    return rope(qn, positions, theta), rope(kn, positions, theta)


# ---------------------------------------------------------------------------
# Attention  ([PATTERN]; [CASE] ingredients 1 and 4; reading R5, R8)
# ---------------------------------------------------------------------------
def attend(q, q_pos, k, k_pos, v, layer_type: str, window: int,
           scale: float | None = None, k_valid=None):
    """Masked softmax attention on absolute positions.

    q: [B, Tq, H, d] with positions q_pos [B, Tq]; k, v: [B, S, G, d] with
    positions k_pos [B, S]; k_valid [B, S] optionally marks usable keys.
    Returns (O [B, Tq, H, d], lse [B, H, Tq]) in float64; lse is the natural
    log of the softmax denominator of the scaled logits.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Tq, H, d = q.shape
    G = k.shape[2]
    R = H // G
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    mask = allowed(np.asarray(q_pos)[:, :, None], np.asarray(k_pos)[:, None, :],
                   layer_type, window)
    if k_valid is not None:
        mask = mask & np.asarray(k_valid, dtype=bool)[:, None, :]
    out = np.zeros((B, Tq, H, d), dtype=np.float64)
    lse = np.zeros((B, H, Tq), dtype=np.float64)
    for h in range(H):
        g = h // R
        logits = np.einsum("btd,bsd->bts", q[:, :, h], k[:, :, g]) * scale
        logits = np.where(mask, logits, -np.inf)
        mx = logits.max(axis=-1, keepdims=True)
        e = np.exp(logits - mx)
        den = e.sum(axis=-1, keepdims=True)
        out[:, :, h] = np.einsum("bts,bsd->btd", e / den, v[:, :, g])
        lse[:, h] = (mx + np.log(den))[..., 0]
    return out, lse


def prefill_attention(q, k, v, layer_type: str, window: int,
                      scale: float | None = None, rows=None):
    """Prefill: every token of a fresh sequence attends over the same sequence.

    q: [B, T, H, d], k, v: [B, T, G, d] (positions 0 .. T-1).  ``rows`` selects
    a subset of query rows (for sampled checks at large T).
    """
    q = np.asarray(q)
    B, T = q.shape[:2]
    pos = np.broadcast_to(np.arange(T)[None, :], (B, T))
    if rows is None:
        rows = np.arange(T)
    rows = np.asarray(rows)
    return attend(q[:, rows], pos[:, rows], k, pos, v, layer_type, window, scale)


def qkv_projection(x, w_qkv, gain_q, gain_k, positions, H: int, G: int, d: int,
                   eps: float = 1e-6, theta: float = 500000.0, inv_freq=None, out_scale: float = 1.0):
    """[CASE] ingredient 1 (bias-free Q, K and V projections; the block's input x
    is not normed first, ingredient 6) followed by ingredients 2 and 3.

    x: [B, T, D]; w_qkv: [(H + 2G) d, D], rows of W_q, then W_k, then W_v;
    positions [B, T].  inv_freq / out_scale, when given, replace plain RoPE
    (YaRN on full layers, see qk_norm_rope_with).  Returns (q_hat [B, T, H, d],
    k_hat [B, T, G, d], v [B, T, G, d]) in float64.
    """
    x = np.asarray(x, dtype=np.float64)
    B, T, _ = x.shape
    y = x @ np.asarray(w_qkv, dtype=np.float64).T
    q = y[..., :H * d].reshape(B, T, H, d)
    k = y[..., H * d:(H + G) * d].reshape(B, T, G, d)
    v = y[..., (H + G) * d:].reshape(B, T, G, d)
    if inv_freq is None:
        qh, kh = qk_norm_rope(q, k, gain_q, gain_k, positions, eps, theta)
    else:
        qh, kh = qk_norm_rope_with(q, k, gain_q, gain_k, positions, inv_freq, out_scale, eps)
    return qh, kh, v


def out_proj_postnorm_residual(x, attn, w_o, gain, eps: float = 1e-6):
    """[CASE] ingredients 1 and 6: the bias-free output projection, then the
    reordered norm h = x + RMSNorm(attn W_o^T) with one gain per model feature.

    x: [M, D] residual stream; attn: [M, H*d] attention output (heads side by
    side); w_o: [D, H*d] (row j maps the attention features to model feature j);
    gain: [D].  Returns h [M, D] in float64.
    """
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(attn, dtype=np.float64) @ np.asarray(w_o, dtype=np.float64).T
    return x + rms_norm(y, gain, eps)


# ---------------------------------------------------------------------------
# KV cache  ([README] "KV Cache Implementation", "Inference Pipeline";
# [SERVING] per-layer-type cache; readings R6, R7)
# ---------------------------------------------------------------------------
class KVCache:
    """The cache of one sequence for one layer.

    Sliding layers: a ring of exactly ``window`` slots, position p in slot
    p mod window.  Full layers: a linear buffer, position p in slot p.
    Rows are appended in position order; each slot remembers its position.
    """

    def __init__(self, layer_type: str, n_slots: int, G: int, d: int):
        self.layer_type = layer_type
        self.n_slots = n_slots
        self.k = np.zeros((n_slots, G, d), dtype=np.float64)
        self.v = np.zeros((n_slots, G, d), dtype=np.float64)
        self.pos = np.full(n_slots, -1, dtype=np.int64)

    def slot(self, p: int) -> int:
        return p % self.n_slots if self.layer_type == SLIDING else p

    def append(self, positions, k_rows, v_rows) -> list[int]:
        slots = []
        for p, kr, vr in zip(positions, k_rows, v_rows):
            s = self.slot(int(p))
            if s >= self.n_slots:
                raise IndexError(f"position {p} beyond capacity {self.n_slots}")
            self.k[s] = kr
            self.v[s] = vr
            self.pos[s] = p
            slots.append(s)
        return slots

    def valid(self) -> np.ndarray:
        return self.pos >= 0


def append_slots(pos_offset, T: int, layer_type: str, n_slots: int) -> np.ndarray:
    """Slot of each appended token, or -1 when a later token of the same call
    lands in the same slot (so its row does not survive the call).

    pos_offset: [B] first position of the call; returns int64 [B, T].
    """
    pos_offset = np.asarray(pos_offset, dtype=np.int64)
    B = pos_offset.shape[0]
    out = np.empty((B, T), dtype=np.int64)
    for b in range(B):
        slots = [(pos_offset[b] + t) % n_slots if layer_type == SLIDING else pos_offset[b] + t
                 for t in range(T)]
        for t in range(T):
            overwritten = any(slots[u] == slots[t] for u in range(t + 1, T))
            out[b, t] = -1 if overwritten else slots[t]
    return out


def decode_attention(q_hat, caches, q_pos, layer_type: str, window: int,
                     scale: float | None = None):
    """One decode token per sequence over its cache.

    q_hat: [B, H, d] (already normed and rotated); caches: list of B KVCache;
    q_pos: [B] position of the new token (its row is already appended).
    Returns (O [B, H, d], lse [B, H]).
    """
    q_hat = np.asarray(q_hat, dtype=np.float64)
    B, H, d = q_hat.shape
    outs, lses = [], []
    for b in range(B):
        c = caches[b]
        o, lse = attend(q_hat[b][None, None], np.array([[q_pos[b]]]),
                        c.k[None], c.pos[None], c.v[None], layer_type, window,
                        scale, k_valid=c.valid()[None])
        outs.append(o[0, 0])
        lses.append(lse[0, :, 0])
    return np.stack(outs), np.stack(lses)


def chunk_attention(q_hat, k_hat, v, caches, pos_offset, layer_type: str, window: int,
                    scale: float | None = None):
    """A chunk of T new tokens per sequence (positions pos_offset[b] + t) attends
    over what its cache holds before the chunk plus the chunk itself.

    q_hat: [B, T, H, d]; k_hat, v: [B, T, G, d] (already normed / rotated);
    caches: list of B KVCache holding positions < pos_offset[b] (not yet updated).
    Returns (O [B, T, H, d], lse [B, H, T]).
    """
    q_hat = np.asarray(q_hat, dtype=np.float64)
    B, T = q_hat.shape[:2]
    outs, lses = [], []
    for b in range(B):
        c = caches[b]
        keep = c.valid()
        p = int(pos_offset[b]) + np.arange(T)
        k_all = np.concatenate([c.k[keep], np.asarray(k_hat[b], dtype=np.float64)])[None]
        v_all = np.concatenate([c.v[keep], np.asarray(v[b], dtype=np.float64)])[None]
        kp = np.concatenate([c.pos[keep], p])[None]
        o, lse = attend(q_hat[b][None], p[None], k_all, kp, v_all, layer_type, window, scale)
        outs.append(o[0])
        lses.append(lse[0])
    return np.stack(outs), np.stack(lses)


def full_recompute_last_row(q_hat_all, k_hat_all, v_all, layer_type: str,
                            window: int, scale: float | None = None):
    """Last row of the prefill formula over all tokens so far ([B, H, d])."""
    q_hat_all = np.asarray(q_hat_all)
    T = q_hat_all.shape[1]
    o, _ = prefill_attention(q_hat_all, k_hat_all, v_all, layer_type, window,
                             scale, rows=[T - 1])
    return o[:, 0]


# ---------------------------------------------------------------------------
# Cache sizing  ([SERVING] "KV OVERPAY FOR THIS CHECKPOINT"; [CASE] ingredient 4)
# ---------------------------------------------------------------------------
def kv_bytes_per_token(n_layers: int, G: int, d: int, elem_bytes: int = 2) -> int:
    """Naive cache bytes per token when every layer keeps every key and value."""
    return n_layers * G * d * 2 * elem_bytes


def kv_cache_bytes(types: list[str], G: int, d: int, context: int, window: int,
                   elem_bytes: int = 2) -> int:
    """Bytes one sequence of ``context`` tokens holds when sliding layers keep
    only the last ``window`` tokens."""
    per_tok_layer = G * d * 2 * elem_bytes
    return sum(per_tok_layer * (min(context, window) if ty == SLIDING else context)
               for ty in types)
