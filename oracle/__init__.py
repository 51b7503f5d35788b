"""fp64 CPU oracle for the batch-1 Llama decode step, and the brute-force
checkers that pin it.

TEST INFRASTRUCTURE ONLY: the tests, the bench's ``cpu_baseline`` leg and
``__graft_entry__.smoke()`` may use this package; the product path
(``persistent_megakernel_decode_cta_b200``) never imports it, and this package
never imports the product.  It shares nothing with the CUDA path except the
seeded inputs from ``synth_inputs``.

* ``OracleModel``: ctypes wrapper around ``amk_oracle.c`` (fp64 decode step
  with a bf16 KV cache).
* ``brute``: a pure-Python, non-incremental full-sequence forward (numpy) that
  pins the oracle's incremental decode on small configs.
* ``interleave``: a brute-force interleaving checker for task schedules that
  pins the schedule validator.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import numpy as np

from . import build as _build

_LIB: Optional[ctypes.CDLL] = None

_u16p = ctypes.POINTER(ctypes.c_uint16)
_dp = ctypes.POINTER(ctypes.c_double)
_vp = ctypes.c_void_p


class OrcConfig(ctypes.Structure):
    _fields_ = [
        ("hidden", ctypes.c_int32), ("n_layers", ctypes.c_int32),
        ("n_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("ffn", ctypes.c_int32),
        ("vocab", ctypes.c_int32), ("max_ctx", ctypes.c_int32),
        ("rms_eps", ctypes.c_double), ("rope_theta", ctypes.c_double),
        ("tied", ctypes.c_int32), ("quant", ctypes.c_int32),
    ]


_PTR_ARRAYS = ("attn_norm", "ffn_norm", "wq", "wk", "wv", "wo", "wgate",
               "wup", "wdown", "sq", "sk", "sv", "so", "sgate", "sup", "sdown")


class OrcWeights(ctypes.Structure):
    _fields_ = [("embed", _vp), ("final_norm", _vp), ("lm_head", _vp),
                ("lm_head_scale", _vp)] + [(n, ctypes.POINTER(_vp))
                                           for n in _PTR_ARRAYS]


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load (building first if needed) the oracle library.  A ``path`` loads
    another build of the same source (used by the mutation tests)."""
    global _LIB
    if path is None and _LIB is not None:
        return _LIB
    lib = ctypes.CDLL(path or _build.build())
    lib.orc_bf16_to_double.restype = ctypes.c_double
    lib.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.orc_fp16_to_double.restype = ctypes.c_double
    lib.orc_fp16_to_double.argtypes = [ctypes.c_uint16]
    lib.orc_double_to_bf16.restype = ctypes.c_uint16
    lib.orc_double_to_bf16.argtypes = [ctypes.c_double]
    lib.orc_rmsnorm.argtypes = [_dp, _u16p, ctypes.c_int32, ctypes.c_double, _dp]
    lib.orc_matvec.argtypes = [_vp, _u16p, ctypes.c_int32, ctypes.c_int32,
                               ctypes.c_int32, _dp, _dp]
    lib.orc_rope.argtypes = [_dp, ctypes.c_int32, ctypes.c_int32, ctypes.c_double]
    lib.orc_attention_head.argtypes = [_dp, _u16p, _u16p, ctypes.c_int32,
                                       ctypes.c_int32, _dp, _dp]
    lib.orc_silu.restype = ctypes.c_double
    lib.orc_silu.argtypes = [ctypes.c_double]
    lib.orc_argmax.restype = ctypes.c_int32
    lib.orc_argmax.argtypes = [_dp, ctypes.c_int32]
    lib.orc_decode_step.restype = ctypes.c_int32
    lib.orc_decode_step.argtypes = [ctypes.POINTER(OrcConfig),
                                    ctypes.POINTER(OrcWeights), _u16p,
                                    ctypes.c_int32, ctypes.c_int32, _dp,
                                    ctypes.POINTER(ctypes.c_int32), _dp]
    lib.orc_set_threads.restype = ctypes.c_int32
    lib.orc_set_threads.argtypes = [ctypes.c_int32]
    if path is None:
        _LIB = lib
    return lib


# ---- numpy helpers ---------------------------------------------------------

def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray, typ=None):
    p = a.ctypes.data_as(typ) if typ is not None else ctypes.c_void_p(a.ctypes.data)
    return p


def to_numpy_bits(t) -> np.ndarray:
    """A torch bf16/fp16 tensor -> its uint16 bits; int8 -> int8 and packed
    int4 (uint8) -> uint8 (CPU)."""
    import torch
    t = t.detach().to("cpu").contiguous()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype in (torch.int8, torch.uint8):
        return t.numpy()
    raise TypeError(f"unexpected weight dtype {t.dtype}")


# ---- single-op entry points (used by the pin tests) ------------------------

def bf16_to_double(bits: int, lib=None) -> float:
    return (lib or load()).orc_bf16_to_double(int(bits))


def fp16_to_double(bits: int, lib=None) -> float:
    return (lib or load()).orc_fp16_to_double(int(bits))


def double_to_bf16(v: float, lib=None) -> int:
    return int((lib or load()).orc_double_to_bf16(float(v)))


def rmsnorm(x, g_bits, eps: float, lib=None) -> np.ndarray:
    x = _f64(x)
    g = np.ascontiguousarray(g_bits, dtype=np.uint16)
    out = np.zeros_like(x)
    (lib or load()).orc_rmsnorm(_ptr(x, _dp), _ptr(g, _u16p), len(x), eps,
                                _ptr(out, _dp))
    return out


def matvec(W, x, scale_bits=None, lib=None) -> np.ndarray:
    """W: uint16 bf16 bits [rows, cols], int8 [rows, cols] with fp16 bits
    ``scale_bits`` [rows], or packed int4 uint8 [rows, cols / 2] with fp16
    bits ``scale_bits`` [rows, ceil(cols / 128)] (cols = len(x))."""
    W = np.ascontiguousarray(W)
    x = _f64(x)
    rows, cols = W.shape
    y = np.zeros(rows, dtype=np.float64)
    quant = {np.dtype(np.uint16): 0, np.dtype(np.int8): 1, np.dtype(np.uint8): 2}.get(W.dtype)
    if quant is None:
        raise TypeError("bf16 weights are passed as uint16 bits")
    if quant == 2:
        cols = len(x)
        if W.shape[1] * 2 != cols:
            raise ValueError("packed int4 rows hold len(x) / 2 bytes")
    s = None
    if quant:
        s = np.ascontiguousarray(scale_bits, dtype=np.uint16)
    (lib or load()).orc_matvec(_ptr(W), _ptr(s, _u16p) if s is not None else None,
                               quant, rows, cols, _ptr(x, _dp), _ptr(y, _dp))
    return y


def rope(v, pos: int, theta: float, lib=None) -> np.ndarray:
    v = _f64(v).copy()
    (lib or load()).orc_rope(_ptr(v, _dp), len(v), int(pos), float(theta))
    return v


def attention_head(q, K_bits, V_bits, lib=None):
    """Returns (out[hd], probs[npos]) for one query head over bf16 rows."""
    q = _f64(q)
    K = np.ascontiguousarray(K_bits, dtype=np.uint16)
    V = np.ascontiguousarray(V_bits, dtype=np.uint16)
    npos, hd = K.shape
    out = np.zeros(hd, dtype=np.float64)
    probs = np.zeros(max(npos, 1), dtype=np.float64)
    (lib or load()).orc_attention_head(_ptr(q, _dp), _ptr(K, _u16p),
                                       _ptr(V, _u16p), npos, hd,
                                       _ptr(out, _dp), _ptr(probs, _dp))
    return out, probs[:npos]


def silu(z: float, lib=None) -> float:
    return (lib or load()).orc_silu(float(z))


def argmax(v, lib=None) -> int:
    v = _f64(v)
    return int((lib or load()).orc_argmax(_ptr(v, _dp), len(v)))


def set_threads(n: int = 0, lib=None) -> int:
    """Set the OpenMP thread count (0 keeps it); returns the count in use."""
    return int((lib or load()).orc_set_threads(int(n)))


# ---- the decode step -------------------------------------------------------

class OracleModel:
    """fp64 decode steps over a bf16 KV cache, on the weights made by
    ``synth_inputs.make_model`` (torch tensors on any device; they are copied
    to host memory once)."""

    def __init__(self, cfg, weights: Dict[str, object], lib=None):
        self.cfg = cfg
        self.lib = lib or load()
        c = OrcConfig()
        c.hidden, c.n_layers = cfg.hidden, cfg.n_layers
        c.n_heads, c.n_kv_heads = cfg.n_heads, cfg.n_kv_heads
        c.head_dim, c.ffn, c.vocab = cfg.head_dim, cfg.ffn, cfg.vocab
        c.max_ctx = cfg.max_ctx
        c.rms_eps, c.rope_theta = cfg.rms_eps, cfg.rope_theta
        c.tied = 1 if cfg.tied else 0
        c.quant = {"bf16": 0, "w8a16": 1, "w4a16": 2}[cfg.quant]
        self._c = c
        self._keep = []  # keeps numpy buffers alive for the C side

        def keep(t):
            a = to_numpy_bits(t)
            self._keep.append(a)
            return ctypes.c_void_p(a.ctypes.data)

        w = OrcWeights()
        w.embed = keep(weights["embed"])
        w.final_norm = keep(weights["final_norm"])
        w.lm_head = keep(weights["lm_head"]) if weights["lm_head"] is not None else None
        w.lm_head_scale = (keep(weights["lm_head_scale"])
                           if weights.get("lm_head_scale") is not None else None)
        L = cfg.n_layers
        for name in _PTR_ARRAYS:
            lst = weights.get(name)
            arr = (_vp * L)()
            if lst is not None:
                for i, t in enumerate(lst):
                    arr[i] = keep(t)
            self._keep.append(arr)
            setattr(w, name, ctypes.cast(arr, ctypes.POINTER(_vp)))
        self._w = w
        self.kv = np.zeros((L, 2, cfg.n_kv_heads, cfg.max_ctx, cfg.head_dim),
                           dtype=np.uint16)

    def reset(self):
        self.kv[...] = 0

    def fill_kv(self, kv_rows) -> None:
        """Copy bf16 rows [L, 2, nkv, ctx, hd] into positions 0..ctx-1."""
        a = to_numpy_bits(kv_rows) if not isinstance(kv_rows, np.ndarray) else kv_rows
        ctx = a.shape[3]
        self.kv[:, :, :, :ctx, :] = a

    def step(self, token: int, pos: int, trace: bool = False):
        """One decode step.  Returns (logits float64 [vocab], argmax, trace)
        where trace is [n_layers, 2, hidden] (residual after attention and
        after the FFN) or None."""
        cfg = self.cfg
        logits = np.zeros(cfg.vocab, dtype=np.float64)
        am = ctypes.c_int32(-1)
        tr = np.zeros((cfg.n_layers, 2, cfg.hidden)) if trace else None
        rc = self.lib.orc_decode_step(
            ctypes.byref(self._c), ctypes.byref(self._w),
            self.kv.ctypes.data_as(_u16p), int(token), int(pos),
            logits.ctypes.data_as(_dp), ctypes.byref(am),
            tr.ctypes.data_as(_dp) if tr is not None else None)
        if rc != 0:
            raise ValueError(f"oracle rejected token={token} pos={pos}")
        return logits, int(am.value), tr

    def greedy(self, prompt, n_new: int, start_pos: int = 0):
        """Feeds ``prompt`` then decodes ``n_new`` greedy tokens.  Returns
        (tokens generated, list of logits for each generated token)."""
        pos = start_pos
        out_tokens, out_logits = [], []
        logits, am = None, None
        for t in prompt:
            logits, am, _ = self.step(t, pos)
            pos += 1
        for _ in range(n_new):
            out_tokens.append(am)
            out_logits.append(logits)
            logits, am, _ = self.step(am, pos)
            pos += 1
        return out_tokens, out_logits
