"""amk_decode_step_noalloc: the decode step for callers that may not allocate
device memory (a plugin whose host framework owns every device byte through
its own allocator, or a loop that cannot afford cudaMalloc's implicit
synchronisation).  The caller brings the weights, the KV cache and the
logits buffer; the step's scratch is the library's fixed static array.

The test calls it through the C ABI twice in a row (positions 0 and 1, so the
second call reads the KV row the first one wrote) and checks logits, greedy
token and KV cache against the allocating entry point amk_decode_step, within
the parity tolerance the other GPU tests use.  This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import persistent_megakernel_decode_cta_b200 as amk
from persistent_megakernel_decode_cta_b200 import abi, build
import synth_inputs as si

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built(cuda_ok):
    build.build()


def _weights_struct(cfg, w):
    """amk_weights for torch tensors; returns the struct and its keep-alive list."""
    s = abi.Weights()
    keep = []
    s.embed = w["embed"].data_ptr()
    s.final_norm = w["final_norm"].data_ptr()
    s.lm_head = w["lm_head"].data_ptr() if w["lm_head"] is not None else None
    s.lm_head_scale = (w["lm_head_scale"].data_ptr()
                       if w.get("lm_head_scale") is not None else None)
    for name in amk.Decoder._PER_LAYER:
        lst = w.get(name)
        if lst is None:
            continue
        arr = (ctypes.c_void_p * cfg.n_layers)(*[t.data_ptr() for t in lst])
        keep.append(arr)
        setattr(s, name, ctypes.cast(arr, abi.c_vpp))
    return s, keep


@pytest.mark.parametrize("name", ["tiny", "tiny_w8", "smol135"])
def test_noalloc_matches_allocating_entry_point(name):
    cfg = (si.get_config("tiny").with_(quant="w8a16", name="tiny_w8") if name == "tiny_w8"
           else si.get_config(name))
    w = si.make_model(cfg, device="cuda")
    toks = si.make_prompt(cfg, 2)
    tol = (2e-2 if cfg.quant == "w8a16" else 1e-2)

    # reference: the allocating entry point
    dec = amk.Decoder(cfg, w)
    ref_logits, ref_tok = [], []
    lg = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    for pos, t in enumerate(toks):
        ref_tok.append(dec.step(t, pos, logits=lg))
        ref_logits.append(lg.clone())
    ref_kv = [torch.stack(dec.kv(l))[:, :, :2].clone() for l in range(cfg.n_layers)]
    dec.close()

    # the no-allocation entry point: caller-owned KV cache and logits
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    plan = amk.Plan(cfg, sms)
    ws, keep = _weights_struct(cfg, w)
    kv = torch.zeros((cfg.n_layers, 2, cfg.n_kv_heads, cfg.max_ctx, cfg.head_dim),
                     dtype=torch.bfloat16, device="cuda")
    out = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    lib = abi.lib()
    for pos, t in enumerate(toks):
        am = ctypes.c_int32(-1)
        rc = lib.amk_decode_step_noalloc(plan._p, ctypes.byref(ws), kv.data_ptr(), t, pos,
                                         out.data_ptr(), ctypes.byref(am),
                                         ctypes.c_void_p(stream))
        assert rc == 0, lib.amk_last_error().decode()
        r = ref_logits[pos].double().cpu().numpy()
        g = out.double().cpu().numpy()
        assert np.abs(g - r).max() <= tol * np.abs(r).max()
        assert am.value == ref_tok[pos]
    for l in range(cfg.n_layers):
        got = kv[l, :, :, :2].float()
        assert torch.allclose(got, ref_kv[l].float(), rtol=2 ** -7, atol=1e-6)
    plan.close()


def test_noalloc_rejects_models_beyond_the_static_scratch():
    """A model whose scratch does not fit the static array is refused before
    any GPU work (the pointers below are valid but never read)."""
    big = si.get_config("llama7b").with_(n_layers=120, name="big")  # ~23 MB of scratch
    plan = amk.Plan(big, 148)
    dummy = torch.empty(64, dtype=torch.uint8, device="cuda")
    ptrs = (ctypes.c_void_p * big.n_layers)(*([dummy.data_ptr()] * big.n_layers))
    ws = abi.Weights()
    for f in ("embed", "final_norm", "lm_head"):
        setattr(ws, f, dummy.data_ptr())
    for name in ("attn_norm", "ffn_norm", "wq", "wk", "wv", "wo", "wgate", "wup", "wdown"):
        setattr(ws, name, ctypes.cast(ptrs, abi.c_vpp))
    lib = abi.lib()
    rc = lib.amk_decode_step_noalloc(plan._p, ctypes.byref(ws), dummy.data_ptr(), 0, 0,
                                     dummy.data_ptr(), None, None)
    assert rc == abi.ERR["AMK_ERR_UNSUPPORTED"]
    assert b"static array" in lib.amk_last_error()
    plan.close()
