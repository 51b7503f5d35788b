"""Batch-1 Llama-family decode as one persistent cooperative kernel per token
on B200 (sm_100a), behind the C ABI in include/amk.h.

This module marshals arguments for libamk.so; every step of the decode runs
in the library's kernel.  PyTorch only supplies device memory and the stream.
There is no CPU fallback: without the built library every call raises.
"""
from __future__ import annotations

import ctypes
from typing import Dict, List, Optional, Tuple

from . import abi

__all__ = ["AmkError", "Decoder", "Plan", "validate_graph", "default_options", "version",
           "make_config", "weights_struct", "decode_step_noalloc", "read_ceiling"]


class AmkError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        self.name = abi.STATUS.get(status, str(status))
        super().__init__(f"{self.name}: {message}")


def _check(rc: int, what: str):
    if rc != abi.AMK_OK:
        msg = abi.lib().amk_last_error().decode(errors="replace")
        raise AmkError(rc, f"{what}: {msg}")


def version() -> str:
    return abi.lib().amk_version().decode()


def default_options(**overrides) -> abi.Options:
    o = abi.Options()
    _check(abi.lib().amk_default_options(ctypes.byref(o)), "amk_default_options")
    for k, v in overrides.items():
        setattr(o, k, v)
    return o


def make_config(cfg) -> abi.Config:
    """An amk_config from any object with the shape attributes of
    ``synth_inputs.ModelConfig``."""
    c = abi.Config()
    for f in ("hidden", "n_layers", "n_heads", "n_kv_heads", "head_dim", "ffn", "vocab",
              "max_ctx"):
        setattr(c, f, int(getattr(cfg, f)))
    c.rms_eps = float(cfg.rms_eps)
    c.rope_theta = float(cfg.rope_theta)
    c.tied_embeddings = 1 if cfg.tied else 0
    quant = {"bf16": abi.QUANT_BF16, "w8a16": abi.QUANT_W8A16,
             "w4a16": abi.QUANT_W4A16}.get(cfg.quant)
    if quant is None:
        raise AmkError(abi.ERR["AMK_ERR_UNSUPPORTED"],
                       f"no kernel for weight format {cfg.quant!r}")
    c.quant = quant
    return c


# ---- schedule graphs ---------------------------------------------------------

def _graph_struct(g: Dict) -> Tuple[abi.Graph, list]:
    """Marshals the plain graph format (see oracle/interleave.py) into an
    amk_graph; returns the struct and the arrays that keep it alive."""
    tasks, queues = g["tasks"], g["queues"]
    T = len(tasks)
    gt = (abi.GraphTask * max(T, 1))()
    waits, sigs, accs = [], [], []
    for i, t in enumerate(tasks):
        gt[i].sm = t["sm"]
        gt[i].wait_begin, gt[i].wait_count = len(waits), len(t["waits"])
        waits += t["waits"]
        gt[i].signal_begin, gt[i].signal_count = len(sigs), len(t["signals"])
        sigs += t["signals"]
        gt[i].access_begin, gt[i].access_count = len(accs), len(t["accesses"])
        accs += t["accesses"]
    gw = (abi.GraphWait * max(len(waits), 1))(*[abi.GraphWait(c, th) for c, th in waits])
    gs = (abi.c_i32 * max(len(sigs), 1))(*sigs)
    ga = (abi.GraphAccess * max(len(accs), 1))(*[abi.GraphAccess(*a) for a in accs])
    bufs = g["buffers"]
    gb = (abi.GraphBuffer * max(len(bufs), 1))(
        *[abi.GraphBuffer(b["size"], abi.BUF_OUTPUT if b["output"] else 0, b["pair"])
          for b in bufs])
    off, flat = [0], []
    for q in queues:
        flat += q
        off.append(len(flat))
    go = (abi.c_i32 * len(off))(*off)
    gq = (abi.c_i32 * max(len(flat), 1))(*flat)
    G = abi.Graph()
    G.n_tasks, G.n_counters, G.n_buffers = T, g["n_counters"], len(bufs)
    G.n_sms = len(queues)
    G.n_waits, G.n_signals, G.n_accesses = len(waits), len(sigs), len(accs)
    G.tasks, G.waits, G.signals, G.accesses, G.buffers = gt, gw, gs, ga, gb
    G.queue_offsets, G.queue_tasks = go, gq
    return G, [gt, gw, gs, ga, gb, go, gq]


def validate_graph(g: Dict) -> Tuple[bool, str, str]:
    """Runs the library's static validator.  Returns (accepted, rule, message)."""
    G, keep = _graph_struct(g)
    rep = abi.ValidationReport()
    rc = abi.lib().amk_validate_graph(ctypes.byref(G), ctypes.byref(rep))
    if rc == abi.AMK_OK:
        return True, "ok", ""
    if rc == abi.ERR["AMK_ERR_VALIDATION"]:
        return False, abi.RULES.get(rep.rule, str(rep.rule)), rep.message.decode()
    _check(rc, "amk_validate_graph")
    return False, "?", ""


class Plan:
    """The lowered, validated schedule of one decode step (host only)."""

    def __init__(self, cfg, n_sms: int, options: Optional[abi.Options] = None):
        self._p = ctypes.c_void_p()
        rep = abi.ValidationReport()
        rc = abi.lib().amk_plan_create(ctypes.byref(make_config(cfg)),
                                       ctypes.byref(options) if options else None,
                                       int(n_sms), ctypes.byref(self._p), ctypes.byref(rep))
        _check(rc, "amk_plan_create")

    def graph(self) -> Dict:
        """The plan's task graph in the plain dict format."""
        G = abi.Graph()
        _check(abi.lib().amk_plan_graph(self._p, ctypes.byref(G)), "amk_plan_graph")
        tasks = []
        for i in range(G.n_tasks):
            t = G.tasks[i]
            tasks.append({
                "sm": t.sm,
                "waits": [(G.waits[j].counter, G.waits[j].threshold)
                          for j in range(t.wait_begin, t.wait_begin + t.wait_count)],
                "signals": [G.signals[j]
                            for j in range(t.signal_begin, t.signal_begin + t.signal_count)],
                "accesses": [(G.accesses[j].buffer, G.accesses[j].kind,
                              G.accesses[j].begin, G.accesses[j].end)
                             for j in range(t.access_begin, t.access_begin + t.access_count)],
            })
        queues = [[G.queue_tasks[j] for j in range(G.queue_offsets[s], G.queue_offsets[s + 1])]
                  for s in range(G.n_sms)]
        bufs = [{"size": G.buffers[b].size, "output": bool(G.buffers[b].flags & abi.BUF_OUTPUT),
                 "pair": G.buffers[b].pair} for b in range(G.n_buffers)]
        return {"n_counters": G.n_counters, "buffers": bufs, "tasks": tasks, "queues": queues}

    def stats(self) -> abi.PlanStats:
        """Task and counter counts, resolved schedule knobs, streamed bytes."""
        st = abi.PlanStats()
        _check(abi.lib().amk_plan_get_stats(self._p, ctypes.byref(st)), "amk_plan_get_stats")
        return st

    def task_info(self) -> Tuple[List[int], List[int]]:
        G = abi.Graph()
        _check(abi.lib().amk_plan_graph(self._p, ctypes.byref(G)), "amk_plan_graph")
        n = G.n_tasks
        kind = (abi.c_i32 * max(n, 1))()
        layer = (abi.c_i32 * max(n, 1))()
        _check(abi.lib().amk_plan_task_info(self._p, kind, layer), "amk_plan_task_info")
        return list(kind[:n]), list(layer[:n])

    def pos0(self) -> Optional["Plan"]:
        """The schedule of steps at position 0 (a view owned by this plan), or
        None when the plan was made with pos0_plan = -1."""
        p = abi.lib().amk_plan_pos0(self._p)
        if not p:
            return None
        view = Plan.__new__(Plan)
        view._p = ctypes.c_void_p(p)
        view._owner = self  # keeps the owning plan alive
        return view

    def close(self):
        if self._p and not hasattr(self, "_owner"):
            abi.lib().amk_plan_destroy(self._p)
        self._p = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ---- the decoder -------------------------------------------------------------

class _DevArray:
    """__cuda_array_interface__ view of memory the library owns."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3,
                                         "strides": None}


_PER_LAYER = ("attn_norm", "ffn_norm", "wq", "wk", "wv", "wo", "wgate", "wup", "wdown",
              "sq", "sk", "sv", "so", "sgate", "sup", "sdown")


def weights_struct(cfg, weights: Dict[str, object]):
    """An amk_weights for torch CUDA tensors (the dict of
    ``synth_inputs.make_model``).  Returns (struct, keep-alive list): the
    pointer arrays the struct points into live as long as the list."""
    w = abi.Weights()
    keep = []

    def ptr(t):
        return None if t is None else ctypes.c_void_p(t.data_ptr())

    w.embed = ptr(weights["embed"])
    w.final_norm = ptr(weights["final_norm"])
    w.lm_head = ptr(weights.get("lm_head"))
    w.lm_head_scale = ptr(weights.get("lm_head_scale"))
    L = cfg.n_layers
    for name in _PER_LAYER:
        lst = weights.get(name)
        if lst is None:
            setattr(w, name, None)
            continue
        arr = (ctypes.c_void_p * L)(*[t.data_ptr() for t in lst])
        keep.append(arr)
        setattr(w, name, ctypes.cast(arr, abi.c_vpp))
    return w, keep


def decode_step_noalloc(plan: "Plan", w, kv, token: int, pos: int, logits,
                        want_argmax: bool = False, stream=None) -> Optional[int]:
    """amk_decode_step_noalloc: one decode step that allocates nothing.  ``w``
    from weights_struct; ``kv`` (bf16 [L, 2, n_kv_heads, max_ctx, head_dim])
    and ``logits`` (float32 [vocab]) are caller-owned torch CUDA tensors."""
    import torch
    am = abi.c_i32(-1)
    st = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    rc = abi.lib().amk_decode_step_noalloc(plan._p, ctypes.byref(w), kv.data_ptr(), int(token),
                                           int(pos), logits.data_ptr(),
                                           ctypes.byref(am) if want_argmax else None,
                                           ctypes.c_void_p(st))
    _check(rc, "amk_decode_step_noalloc")
    return int(am.value) if want_argmax else None


def read_ceiling(buf, n_sms: int, stage_bytes: int = 32768, stages: int = 3, reps: int = 5,
                 stream=None) -> float:
    """amk_read_ceiling: GB/s of the decode kernel's bulk-copy weight stream
    with nothing consuming it, over the torch CUDA tensor ``buf`` (>= 1 GiB)."""
    import torch
    g = ctypes.c_double(0.0)
    st = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    rc = abi.lib().amk_read_ceiling(ctypes.c_void_p(buf.data_ptr()),
                                    buf.numel() * buf.element_size(), int(n_sms),
                                    int(stage_bytes), int(stages), int(reps), ctypes.c_void_p(st),
                                    ctypes.byref(g))
    _check(rc, "amk_read_ceiling")
    return g.value


class Decoder:
    """One amk_handle: weights borrowed from torch CUDA tensors, KV cache and
    workspace owned by the library."""

    _PER_LAYER = _PER_LAYER

    def __init__(self, cfg, weights: Dict[str, object], options: Optional[abi.Options] = None,
                 stream=None):
        import torch
        self.cfg = cfg
        self._weights = weights  # keep the borrowed tensors alive
        w, self._keep = weights_struct(cfg, weights)
        if stream is None:
            stream = torch.cuda.current_stream().cuda_stream
        self.stream = stream
        self._h = ctypes.c_void_p()
        rc = abi.lib().amk_create(ctypes.byref(make_config(cfg)), ctypes.byref(w),
                                  ctypes.byref(options) if options else None,
                                  ctypes.c_void_p(stream), ctypes.byref(self._h))
        _check(rc, "amk_create")

    # -- steps
    def step(self, token: int, pos: int, logits=None, want_argmax: bool = True) -> Optional[int]:
        """One decode step (one cooperative launch).  ``logits``: optional torch
        CUDA float32 tensor [vocab] to receive the logits.  Returns the greedy
        token when ``want_argmax`` (this synchronises the stream)."""
        am = abi.c_i32(-1)
        rc = abi.lib().amk_decode_step(self._h, int(token), int(pos),
                                       ctypes.c_void_p(logits.data_ptr()) if logits is not None
                                       else None,
                                       ctypes.byref(am) if want_argmax else None)
        _check(rc, "amk_decode_step")
        return int(am.value) if want_argmax else None

    def step_host(self, token: int, pos: int, logits_host=None) -> int:
        """One step with the logits copied into host memory ``logits_host``
        (a contiguous float32 numpy array or CPU tensor, ideally pinned)."""
        am = abi.c_i32(-1)
        p = None
        if logits_host is not None:
            p = ctypes.c_void_p(logits_host.ctypes.data if hasattr(logits_host, "ctypes")
                                else logits_host.data_ptr())
        rc = abi.lib().amk_decode_step_host(self._h, int(token), int(pos), p, ctypes.byref(am))
        _check(rc, "amk_decode_step_host")
        return int(am.value)

    def reset(self):
        _check(abi.lib().amk_reset_kv(self._h), "amk_reset_kv")

    # -- views of library-owned memory
    def logits(self):
        import torch
        p = ctypes.c_void_p()
        _check(abi.lib().amk_get_logits(self._h, ctypes.byref(p)), "amk_get_logits")
        return torch.as_tensor(_DevArray(p.value, (self.cfg.vocab,), "<f4"), device="cuda")

    def kv(self, layer: int):
        """(K, V) bf16 views [n_kv_heads, max_ctx, head_dim] of one layer's cache."""
        import torch
        k, v = ctypes.c_void_p(), ctypes.c_void_p()
        _check(abi.lib().amk_get_kv(self._h, int(layer), ctypes.byref(k), ctypes.byref(v)),
               "amk_get_kv")
        shape = (self.cfg.n_kv_heads, self.cfg.max_ctx, self.cfg.head_dim)
        kt = torch.as_tensor(_DevArray(k.value, shape, "<i2"), device="cuda").view(torch.bfloat16)
        vt = torch.as_tensor(_DevArray(v.value, shape, "<i2"), device="cuda").view(torch.bfloat16)
        return kt, vt

    def workspace(self) -> Dict[str, object]:
        """fp32 views of the last step's activations: qkv [L, qkv_rows],
        xmid / xout [L, hidden], act [L, ffn] (the values of the flagged
        words; act's with 15 mantissa bits)."""
        import torch
        ws = abi.Workspace()
        _check(abi.lib().amk_get_workspace(self._h, ctypes.byref(ws)), "amk_get_workspace")
        L = self.cfg.n_layers

        def view(p, n):
            w = torch.as_tensor(_DevArray(p, (L, n, 2), "<f4"), device="cuda")
            return w[:, :, 0]

        act = torch.as_tensor(_DevArray(ws.act, (L, self.cfg.ffn), "<i4"), device="cuda")
        act = (act & ~0xFF).view(torch.float32)  # drop the 8-bit tag
        return {"qkv": view(ws.qkv, ws.qkv_rows), "xmid": view(ws.xmid, self.cfg.hidden),
                "xout": view(ws.xout, self.cfg.hidden), "act": act}

    def profile(self):
        """Phase timers of the last step (needs options.profile = 1): a uint64
        numpy array [n_sms, 8 kinds, 8 fields] (see amk_get_profile)."""
        import numpy as np
        n = self.stats().n_sms * 8 * 8
        buf = np.zeros(n, dtype=np.uint64)
        _check(abi.lib().amk_get_profile(self._h, buf.ctypes.data_as(
            ctypes.POINTER(ctypes.c_uint64)), n), "amk_get_profile")
        return buf.reshape(-1, 8, 8)

    def stats(self) -> abi.PlanStats:
        s = abi.PlanStats()
        _check(abi.lib().amk_get_stats(self._h, ctypes.byref(s)), "amk_get_stats")
        return s

    def check_guards(self) -> int:
        """Guards a kernel or copy wrote into (amk_check_guards; needs
        options.debug_checks = 1); 0 when every buffer stayed in bounds."""
        n = abi.c_i32(-1)
        _check(abi.lib().amk_check_guards(self._h, ctypes.byref(n)), "amk_check_guards")
        return int(n.value)

    def error_info(self) -> abi.ErrorInfo:
        e = abi.ErrorInfo()
        _check(abi.lib().amk_get_error_info(self._h, ctypes.byref(e)), "amk_get_error_info")
        return e

    def close(self):
        if getattr(self, "_h", None):
            abi.lib().amk_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
