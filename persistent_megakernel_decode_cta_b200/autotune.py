"""Schedule-knob search for the decode megakernel on the current device.

The schedule of a step is fixed by a few knobs (README "Two autoresearch
loops": tiling, SM assignment, pipelining depth): GEMV row tiles per SM per
level, the rotation of the tile-to-SM map, the weight ring's stage size and
in-flight cap, the split-K attention chunks, the fused FFN level.  ``tune`` tries a grid of them the way the pages' schedule loop
does -- lower, validate, check, measure, keep or drop -- with a correctness
gate that needs no reference implementation: every candidate is lowered and
validated by ``amk_create`` (a rejected schedule is dropped), and its first
step's logits must equal the default schedule's within ``rtol`` of the
largest logit (all schedules compute the same function; they differ only in
rounding order).  The fastest candidate that passes is returned.

    python -m persistent_megakernel_decode_cta_b200.autotune --model tinyllama --ctx 0

(the command line draws a seeded random-init model of the named shape).
"""
from __future__ import annotations

import itertools
import json
import sys
from typing import Dict, Iterable, List, Optional, Tuple

from . import Decoder, AmkError, default_options

# The pages' schedule knobs: tiling (tasks_per_sm: GEMV row tiles per SM per
# level), SM assignment (sm_rotate), pipelining depth (the ring's stages and
# stage size, the in-flight cap), fusion grouping (ffn_fused) and the
# split-K attention chunks.
DEFAULT_SPACE: Dict[str, List[int]] = {
    "stage_bytes": [32768, 49152, 65536],  # ring_stages 0: as many as make 192 KiB
    "attn_splits": [0, 2, 8],
    "ffn_fused": [1, 2, -1],
    "tasks_per_sm": [1, 2],
    "sm_rotate": [0, 37],
    "inflight_kb": [0, 96],
}


def _candidates(space: Dict[str, Iterable[int]]) -> List[Dict[str, int]]:
    keys = list(space)
    return [dict(zip(keys, vals)) for vals in itertools.product(*(list(space[k]) for k in keys))]


def _time_steps(dec: Decoder, ctx: int, steps: int, warmup: int) -> float:
    import torch
    for _ in range(warmup):
        dec.step(-1, ctx, want_argmax=False)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(steps):
        dec.step(-1, ctx, want_argmax=False)
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) * 1e3 / steps


def tune(cfg, weights, ctx: int = 0, kv=None, space: Optional[Dict[str, Iterable[int]]] = None,
         steps: int = 20, warmup: int = 3, token: int = 0,
         rtol: Optional[float] = None) -> Tuple[object, List[Dict]]:
    """Returns (the fastest passing amk_options, one report row per candidate:
    knobs, status "ok" / "rejected: ..." / "mismatch", us per step, max |dlogit|).

    cfg/weights are as for Decoder; kv, if given, is the cache content for
    positions 0..ctx-1 as a [n_layers, 2, n_kv_heads, ctx, head_dim] bf16
    tensor on the device."""
    import torch

    if rtol is None:
        # bf16 schedules differ only in rounding order; int8 / int4 GEMVs
        # quantise each lane's activations to int16 with the lane's own
        # scale, and a different K split moves those grids (both stay within
        # the 2e-2 parity bound of the exact step)
        rtol = 1e-3 if getattr(cfg, "quant", "bf16") == "bf16" else 1e-2

    def make(opts):
        dec = Decoder(cfg, weights, opts)
        if kv is not None and ctx:
            for layer in range(cfg.n_layers):
                k, v = dec.kv(layer)
                k[:, :ctx].copy_(kv[layer, 0])
                v[:, :ctx].copy_(kv[layer, 1])
        return dec

    logits = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    ref_dec = make(default_options())
    ref_dec.step(token, ctx, logits=logits)
    ref = logits.clone()
    scale = float(ref.abs().max())
    best, best_us, rows = default_options(), _time_steps(ref_dec, ctx, steps, warmup), []
    ref_dec.close()
    rows.append({"knobs": {}, "status": "ok", "us": best_us, "max_dlogit": 0.0})
    for knobs in _candidates(space or DEFAULT_SPACE):
        opts = default_options(**knobs)
        try:
            dec = make(opts)
        except AmkError as e:
            rows.append({"knobs": knobs, "status": f"rejected: {e.name}", "us": None,
                         "max_dlogit": None})
            continue
        try:
            dec.step(token, ctx, logits=logits)
            err = float((logits - ref).abs().max())
            if not err <= rtol * scale:
                rows.append({"knobs": knobs, "status": "mismatch", "us": None,
                             "max_dlogit": err})
                continue
            us = _time_steps(dec, ctx, steps, warmup)
            rows.append({"knobs": knobs, "status": "ok", "us": us, "max_dlogit": err})
            if us < best_us:
                best, best_us = opts, us
        finally:
            dec.close()
    return best, rows


def main(argv=None) -> int:
    import argparse
    import os
    import torch

    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--model", default="tinyllama")
    ap.add_argument("--ctx", type=int, default=0)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--space", default=None, help="JSON {knob: [values]}")
    args = ap.parse_args(argv)
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import synth_inputs as si  # seeded random-init weights of a named shape
    cfg = si.get_config(args.model)
    w = si.make_model(cfg, seed=0, device="cuda")
    kv = si.make_kv_fill(cfg, args.ctx, device="cuda") if args.ctx else None
    space = json.loads(args.space) if args.space else None
    best, rows = tune(cfg, w, args.ctx, kv, space, steps=args.steps)
    for r in sorted(rows, key=lambda r: (r["us"] is None, r["us"] or 0)):
        print(json.dumps(r))
    fields = [f for f, _ in best._fields_ if f != "reserved"]
    print(json.dumps({"best": {f: getattr(best, f) for f in fields}}))
    return 0


if __name__ == "__main__":
    sys.exit(main())
