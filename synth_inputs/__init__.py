"""Seeded synthetic inputs for the batch-1 Llama decode step.

This module is shared by the oracle tests, the CUDA-path tests and the bench.
It only draws random numbers and lays them out; it holds none of the decode
step's arithmetic (no norm, matvec, RoPE, attention or softmax).

Recipe (the pages run random-init models of published shapes; no trained
weights are needed or used):

* linear and embedding weights: N(0, 0.02) drawn in fp32, rounded to bf16
  (round-to-nearest-even, which is what ``torch.Tensor.to(torch.bfloat16)``
  does);
* RMSNorm gains: 1 + N(0, 0.01), rounded to bf16, so that a dropped gain
  multiply cannot hide behind gains equal to one;
* W8A16 weights: from the same N(0, 0.02) fp32 masters, one symmetric scale
  per output row, ``s = fp16(max|w_row| / 127)`` and
  ``q = clamp(round_half_even(w / s), -127, 127)`` (a row of zeros gets s = 1,
  q = 0).  The decode step consumes q and s; neither side re-quantises;
* W4A16 weights: from the same masters, one symmetric scale per group of
  ``INT4_GROUP`` consecutive inputs of a row (the last group of a row is
  shorter when the row length is not a multiple of it),
  ``s = fp16(max|w_group| / 7)`` and ``q = clamp(round_half_even(w / s), -7, 7)``
  (an all-zero group gets s = 1, q = 0).  Codes are packed two per byte in
  4-bit two's complement, input 2i in the low nibble of byte i and input
  2i + 1 in the high nibble; scales are fp16 [rows][ceil(cols / INT4_GROUP)];
* prompt token ids: uniform in [0, vocab);
* synthetic KV-cache fill for long contexts: N(0, 1) rounded to bf16.

Every tensor is drawn from its own generator whose seed is derived from the
base seed and the tensor's name, so the bytes do not depend on the order in
which tensors are made.  The same call on the same device type gives the same
bytes; CPU and CUDA generators give different (equally valid) bytes, so a test
draws once and hands the identical bytes to both sides.
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Dict, List, Optional

import torch

__all__ = [
    "ModelConfig",
    "CONFIGS",
    "get_config",
    "make_model",
    "make_prompt",
    "make_kv_fill",
    "model_bytes",
    "streamed_weight_bytes",
]


@dataclasses.dataclass(frozen=True)
class ModelConfig:
    name: str
    hidden: int
    n_layers: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    max_ctx: int
    rms_eps: float = 1e-5
    rope_theta: float = 1e4
    tied: bool = False
    quant: str = "bf16"  # "bf16", "w8a16" or "w4a16"

    @property
    def q_rows(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def kv_rows(self) -> int:
        return self.n_kv_heads * self.head_dim

    def with_(self, **kw) -> "ModelConfig":
        return dataclasses.replace(self, **kw)


# The five workloads: a tiny decoder, then random-init models shaped like
# SmolLM2-135M, TinyLlama-1.1B, Llama-1B (W8A16) and Llama-7B (bf16 and W8A16).
CONFIGS: Dict[str, ModelConfig] = {
    "tiny": ModelConfig("tiny", 64, 2, 4, 2, 16, 172, 256, max_ctx=32),
    "smol135": ModelConfig("smol135", 576, 30, 9, 3, 64, 1536, 49152,
                           max_ctx=256, tied=True),
    "tinyllama": ModelConfig("tinyllama", 2048, 22, 32, 4, 64, 5632, 32000,
                             max_ctx=1088),
    "llama1b_w8": ModelConfig("llama1b_w8", 2048, 16, 32, 8, 64, 8192, 128256,
                              max_ctx=576, quant="w8a16"),
    "llama7b": ModelConfig("llama7b", 4096, 32, 32, 32, 128, 11008, 32000,
                           max_ctx=2112),
    "llama7b_w8": ModelConfig("llama7b_w8", 4096, 32, 32, 32, 128, 11008,
                              32000, max_ctx=2112, quant="w8a16"),
    # int4 weight-only variants (the pages' int4 figure is on SmolLM2-135M)
    "smol135_w4": ModelConfig("smol135_w4", 576, 30, 9, 3, 64, 1536, 49152,
                              max_ctx=256, tied=True, quant="w4a16"),
    "llama7b_w4": ModelConfig("llama7b_w4", 4096, 32, 32, 32, 128, 11008,
                              32000, max_ctx=2112, quant="w4a16"),
}


def get_config(name_or_cfg) -> ModelConfig:
    if isinstance(name_or_cfg, ModelConfig):
        return name_or_cfg
    return CONFIGS[name_or_cfg]


def _seed_for(seed: int, name: str) -> int:
    h = hashlib.sha256(f"{seed}/{name}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(device, seed: int, name: str) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed_for(seed, name))
    return g


def _normal(shape, std, device, seed, name) -> torch.Tensor:
    g = _gen(device, seed, name)
    return torch.randn(shape, generator=g, device=device,
                       dtype=torch.float32).mul_(std)


def _bf16_normal(shape, std, device, seed, name) -> torch.Tensor:
    return _normal(shape, std, device, seed, name).to(torch.bfloat16)


def _gain(n, device, seed, name) -> torch.Tensor:
    return (_normal((n,), 0.01, device, seed, name) + 1.0).to(torch.bfloat16)


def _int8_rows(shape, device, seed, name):
    """Per-output-row symmetric int8 weights from N(0, 0.02) fp32 masters."""
    w = _normal(shape, 0.02, device, seed, name)
    amax = w.abs().amax(dim=1)
    s = (amax / 127.0).to(torch.float16)
    s = torch.where(amax == 0, torch.ones_like(s), s)
    q = torch.round(w / s.to(torch.float32)[:, None]).clamp_(-127, 127)
    q = torch.where((amax == 0)[:, None], torch.zeros_like(q), q)
    del w
    return q.to(torch.int8), s


INT4_GROUP = 128  # inputs per W4A16 scale


def _int4_groups(shape, device, seed, name):
    """Per-group symmetric int4 weights from N(0, 0.02) fp32 masters, packed
    two codes per byte (even input in the low nibble)."""
    rows, cols = shape
    if cols % 2:
        raise ValueError("W4A16 rows need an even number of inputs")
    w = _normal(shape, 0.02, device, seed, name)
    ng = (cols + INT4_GROUP - 1) // INT4_GROUP
    pad = ng * INT4_GROUP - cols
    wp = torch.nn.functional.pad(w, (0, pad)).view(rows, ng, INT4_GROUP)
    amax = wp.abs().amax(dim=2)
    s = (amax / 7.0).to(torch.float16)
    s = torch.where(amax == 0, torch.ones_like(s), s)
    q = torch.round(wp / s.to(torch.float32)[:, :, None]).clamp_(-7, 7)
    q = torch.where((amax == 0)[:, :, None], torch.zeros_like(q), q)
    q = q.view(rows, ng * INT4_GROUP)[:, :cols].to(torch.int16)
    del w, wp
    nib = q & 0xF  # 4-bit two's complement
    packed = (nib[:, 0::2] | (nib[:, 1::2] << 4)).to(torch.uint8)
    return packed, s


def make_model(cfg, seed: int = 0, device="cpu") -> Dict[str, object]:
    """Random-init weights of ``cfg``'s shape.

    Returns a dict with tensors on ``device``:
      embed [vocab, hidden] bf16; final_norm [hidden] bf16;
      lm_head [vocab, hidden] bf16 or int8, or packed int4 [vocab, hidden/2]
      (None when tied);
      lm_head_scale [vocab] fp16 (W8A16), [vocab, groups] fp16 (W4A16), or
      None (bf16 or tied);
      per-layer lists attn_norm, ffn_norm [hidden] bf16;
      wq [nh*hd, hidden], wk/wv [nkv*hd, hidden], wo [hidden, nh*hd],
      wgate/wup [ffn, hidden], wdown [hidden, ffn] (bf16, int8, or packed
      int4 uint8 [out, in/2]), and for W8A16 the fp16 row scales sq, sk, sv,
      so, sgate, sup, sdown ([out]; W4A16: group scales [out, groups]).
    All weights are row-major [out, in].
    """
    cfg = get_config(cfg)
    h, L = cfg.hidden, cfg.n_layers
    if cfg.quant not in ("bf16", "w8a16", "w4a16"):
        raise ValueError(f"unknown quant {cfg.quant!r}")
    qfn = {"w8a16": _int8_rows, "w4a16": _int4_groups}.get(cfg.quant)
    m: Dict[str, object] = {}
    m["embed"] = _bf16_normal((cfg.vocab, h), 0.02, device, seed, "embed")
    m["final_norm"] = _gain(h, device, seed, "final_norm")
    m["lm_head"] = None
    m["lm_head_scale"] = None
    if not cfg.tied:
        if qfn:
            m["lm_head"], m["lm_head_scale"] = qfn((cfg.vocab, h), device, seed, "lm_head")
        else:
            m["lm_head"] = _bf16_normal((cfg.vocab, h), 0.02, device, seed,
                                        "lm_head")
    shapes = {
        "wq": (cfg.q_rows, h),
        "wk": (cfg.kv_rows, h),
        "wv": (cfg.kv_rows, h),
        "wo": (h, cfg.q_rows),
        "wgate": (cfg.ffn, h),
        "wup": (cfg.ffn, h),
        "wdown": (h, cfg.ffn),
    }
    for key in ("attn_norm", "ffn_norm", *shapes):
        m[key] = []
    for key in shapes:
        m["s" + key[1:]] = [] if qfn else None
    for layer in range(L):
        m["attn_norm"].append(_gain(h, device, seed, f"l{layer}.attn_norm"))
        m["ffn_norm"].append(_gain(h, device, seed, f"l{layer}.ffn_norm"))
        for key, shp in shapes.items():
            name = f"l{layer}.{key}"
            if qfn:
                q, s = qfn(shp, device, seed, name)
                m[key].append(q)
                m["s" + key[1:]].append(s)
            else:
                m[key].append(_bf16_normal(shp, 0.02, device, seed, name))
    return m


def make_prompt(cfg, n: int, seed: int = 1, device="cpu") -> List[int]:
    """``n`` uniform token ids in [0, vocab)."""
    cfg = get_config(cfg)
    g = _gen(device, seed, "prompt")
    t = torch.randint(0, cfg.vocab, (n,), generator=g, device=device)
    return [int(v) for v in t.tolist()]


def make_kv_fill(cfg, ctx: int, seed: int = 2, device="cpu",
                 layers: Optional[int] = None) -> torch.Tensor:
    """Synthetic KV-cache rows 0..ctx-1: bf16 N(0,1), shape
    [n_layers, 2, n_kv_heads, ctx, head_dim] (index 0 = K, 1 = V)."""
    cfg = get_config(cfg)
    L = cfg.n_layers if layers is None else layers
    shape = (L, 2, cfg.n_kv_heads, ctx, cfg.head_dim)
    return _bf16_normal(shape, 1.0, device, seed, "kvfill")


def model_bytes(cfg) -> Dict[str, int]:
    """Byte counts of the stored weights (for roofline bookkeeping)."""
    cfg = get_config(cfg)
    h, L = cfg.hidden, cfg.n_layers
    # (rows, inputs) of every linear weight of one layer
    mats = [(cfg.q_rows, h), (cfg.kv_rows, h), (cfg.kv_rows, h), (h, cfg.q_rows),
            (cfg.ffn, h), (cfg.ffn, h), (h, cfg.ffn)]

    def wbytes(rows, cols):  # (weight bytes, scale bytes) of one matrix
        if cfg.quant == "w8a16":
            return rows * cols, rows * 2
        if cfg.quant == "w4a16":
            return rows * cols // 2, rows * ((cols + INT4_GROUP - 1) // INT4_GROUP) * 2
        return rows * cols * 2, 0

    linear = L * sum(wbytes(r, k)[0] for r, k in mats)
    scales = L * sum(wbytes(r, k)[1] for r, k in mats)
    head, head_scales = (0, 0) if cfg.tied else wbytes(cfg.vocab, h)
    norms = (2 * L + 1) * h * 2
    return {
        "linear": linear, "scales": scales + head_scales, "head": head,
        "norms": norms, "embed_row": h * 2,
        "embed_table": cfg.vocab * h * 2,
    }


def streamed_weight_bytes(cfg) -> int:
    """Weight bytes one decode step reads: every linear weight (and int8 row
    or int4 group scale) once, the LM head -- the whole embedding table when tied --, the
    norm gains and the one embedding row of the input token."""
    b = model_bytes(cfg)
    head = b["embed_table"] if get_config(cfg).tied else b["head"]
    return b["linear"] + b["scales"] + head + b["norms"] + b["embed_row"]
