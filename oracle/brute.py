"""Non-incremental full-sequence forward of the Llama decoder (numpy fp64).

TEST INFRASTRUCTURE ONLY.  This is the pin for the oracle's incremental
decode: it recomputes every position of a token sequence from scratch with a
causal mask (no KV cache, no per-step state), using whole-sequence matrix
products, HF's ``repeat_kv`` head mapping and HF's ``rotate_half`` RoPE
written over arrays.  It shares no code with ``amk_oracle.c``.

The workload stores the KV cache in bf16, so K (after RoPE) and V are rounded
to bf16 (nearest, ties to even) before attention, as the definition says.
Slow by design; meant for configs of a few layers and a few dozen positions.
"""
from __future__ import annotations

from typing import Dict, List

import numpy as np


def bf16_bits_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def fp16_bits_to_f64(bits) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def round_to_bf16(v) -> np.ndarray:
    """Nearest bf16 value (8 significant bits, ties to even) of each element,
    returned as float64 (normal range only, which is all these tests need)."""
    v = np.asarray(v, dtype=np.float64)
    mant, exp = np.frexp(v)              # v = mant * 2**exp, |mant| in [0.5, 1)
    scaled = np.ldexp(mant, 8)           # 8 significant bits left of the point
    return np.ldexp(np.rint(scaled), exp - 8)  # rint: ties to even


def dequant(weights: Dict[str, object], key: str, layer=None) -> np.ndarray:
    """A weight matrix as float64: bf16 bits widened, int8 times its fp16
    row scale, or packed int4 (uint8, two 4-bit two's-complement codes per
    byte, the even input in the low nibble) times the fp16 scale of its group
    of 128 inputs."""
    from . import to_numpy_bits
    t = weights[key] if layer is None else weights[key][layer]
    a = to_numpy_bits(t)
    if a.dtype in (np.int8, np.uint8):
        skey = "lm_head_scale" if key == "lm_head" else "s" + key[1:]
        s = weights[skey] if layer is None else weights[skey][layer]
        sc = fp16_bits_to_f64(to_numpy_bits(s))
        if a.dtype == np.int8:
            return a.astype(np.float64) * sc[:, None]
        nib = np.stack([a & 0xF, a >> 4], axis=-1).reshape(a.shape[0], -1).astype(np.int64)
        codes = np.where(nib >= 8, nib - 16, nib)
        cols = codes.shape[1]
        per_input = np.repeat(sc, 128, axis=1)[:, :cols]
        return codes.astype(np.float64) * per_input
    return bf16_bits_to_f64(a)


def _rmsnorm_rows(X, g, eps):
    return X / np.sqrt(np.mean(X * X, axis=-1, keepdims=True) + eps) * g


def _rope_rows(X, positions, theta):
    """X: [n, heads, hd]; HF: x*cos + rotate_half(x)*sin."""
    hd = X.shape[-1]
    inv_freq = theta ** (-np.arange(0, hd, 2, dtype=np.float64) / hd)
    ang = np.outer(np.asarray(positions, dtype=np.float64), inv_freq)
    emb = np.concatenate([ang, ang], axis=-1)           # [n, hd]
    cos, sin = np.cos(emb)[:, None, :], np.sin(emb)[:, None, :]
    x1, x2 = X[..., : hd // 2], X[..., hd // 2:]
    rot = np.concatenate([-x2, x1], axis=-1)
    return X * cos + rot * sin


def forward_all(cfg, weights: Dict[str, object], tokens: List[int]) -> np.ndarray:
    """Logits [len(tokens), vocab] for every position of ``tokens`` (token i
    at position i), recomputed from scratch with a causal mask."""
    n = len(tokens)
    h, nh, nkv, hd = cfg.hidden, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    from . import to_numpy_bits
    E = bf16_bits_to_f64(to_numpy_bits(weights["embed"]))
    X = E[np.asarray(tokens)]                            # [n, h]
    causal = np.tril(np.ones((n, n), dtype=bool))
    for l in range(cfg.n_layers):
        g1 = bf16_bits_to_f64(to_numpy_bits(weights["attn_norm"][l]))
        U = _rmsnorm_rows(X, g1, cfg.rms_eps)
        Q = (U @ dequant(weights, "wq", l).T).reshape(n, nh, hd)
        K = (U @ dequant(weights, "wk", l).T).reshape(n, nkv, hd)
        V = (U @ dequant(weights, "wv", l).T).reshape(n, nkv, hd)
        Q = _rope_rows(Q, range(n), cfg.rope_theta)
        K = round_to_bf16(_rope_rows(K, range(n), cfg.rope_theta))
        V = round_to_bf16(V)
        rep = nh // nkv
        K = np.repeat(K, rep, axis=1)                    # HF repeat_kv
        V = np.repeat(V, rep, axis=1)
        S = np.einsum("ihd,jhd->hij", Q, K) / np.sqrt(hd)  # [heads, n, n]
        S = np.where(causal[None], S, -np.inf)
        S = S - S.max(axis=-1, keepdims=True)
        P = np.exp(S)
        P = P / P.sum(axis=-1, keepdims=True)
        A = np.einsum("hij,jhd->ihd", P, V).reshape(n, nh * hd)
        X = X + A @ dequant(weights, "wo", l).T
        g2 = bf16_bits_to_f64(to_numpy_bits(weights["ffn_norm"][l]))
        U = _rmsnorm_rows(X, g2, cfg.rms_eps)
        G = U @ dequant(weights, "wgate", l).T
        Up = U @ dequant(weights, "wup", l).T
        Act = G / (1.0 + np.exp(-G)) * Up
        X = X + Act @ dequant(weights, "wdown", l).T
    gf = bf16_bits_to_f64(to_numpy_bits(weights["final_norm"]))
    U = _rmsnorm_rows(X, gf, cfg.rms_eps)
    Wh = E if cfg.tied else dequant(weights, "lm_head")
    return U @ Wh.T


def greedy(cfg, weights, prompt: List[int], n_new: int):
    """Greedy continuation by full recomputation: returns (all tokens, logits
    of every position)."""
    toks = list(prompt)
    for _ in range(n_new):
        logits = forward_all(cfg, weights, toks)
        toks.append(int(np.argmax(logits[-1])))
    return toks, forward_all(cfg, weights, toks)
