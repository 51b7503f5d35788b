"""GPU parity: the megakernel (called through the C ABI) against the fp64
oracle on identical seeded weights, element by element on the logits, and
on greedy tokens wherever the oracle's top-2 margin exceeds the bound.

Workloads: the tiny decoder (8 greedy steps from a 4-token prompt) and
random-init models shaped like SmolLM2-135M, TinyLlama-1.1B, Llama-1B
(W8A16) and Llama-7B (bf16 and W8A16), at KV context 0 and the long contexts
of those workloads (long caches filled with seeded N(0,1) bf16 rows).
"""
import numpy as np
import pytest
import torch

import persistent_megakernel_decode_cta_b200 as amk
from persistent_megakernel_decode_cta_b200 import build
import synth_inputs as si
from parity_helpers import Pair, compare, greedy_teacher_forced

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built(cuda_ok):
    build.build()


@pytest.mark.parametrize("variant", ["bf16", "tied", "w8a16"])
@pytest.mark.parametrize("n_sms", [0, 3])
def test_tiny_greedy(variant, n_sms):
    cfg = si.get_config("tiny")
    if variant == "tied":
        cfg = cfg.with_(tied=True, name="tiny_tied")
    elif variant == "w8a16":
        cfg = cfg.with_(quant="w8a16", name="tiny_w8")
    opts = amk.default_options(n_sms=n_sms) if n_sms else None
    pair = Pair(cfg, options=opts)
    st = pair.dec.stats()  # the ring shape resolved from the weight format
    assert (st.ring_stages, st.stage_bytes) == ((4, 49152) if cfg.quant == "w8a16" else (3, 65536))
    prompt = si.make_prompt(cfg, 4)
    worst, checked = greedy_teacher_forced(pair, prompt, 8)
    assert checked >= 6
    # the KV rows the kernel appended equal the oracle's (bf16 of nearly equal
    # fp32/fp64 values: within one bf16 ulp).  The W8A16 GEMV takes its
    # activations in int16 steps of max|x|/32767, so an element of k may move
    # by up to sum_k |w_jk| * max|x| / 65534 (about 2e-4 on this model) before
    # rounding: an absolute term of 1e-3 * max|K| covers it.
    for l in range(cfg.n_layers):
        k, v = pair.dec.kv(l)
        gk = k[:, :12].float().cpu().numpy()
        from oracle.brute import bf16_bits_to_f64
        rk = bf16_bits_to_f64(pair.orc.kv[l, 0, :, :12])
        atol = 1e-3 * float(np.abs(rk).max()) if cfg.quant == "w8a16" else 1e-6
        assert np.allclose(gk, rk, rtol=2 ** -7, atol=atol)


def test_tiny_w4a16_greedy():
    """int4 weights with 128-input group scales (the down projection's 192
    inputs end in a group of 64), 8 greedy steps against the oracle."""
    cfg = si.get_config("tiny").with_(quant="w4a16", ffn=192, name="tiny_w4")
    pair = Pair(cfg)
    st = pair.dec.stats()
    assert (st.ring_stages, st.stage_bytes) == (4, 49152)
    worst, checked = greedy_teacher_forced(pair, si.make_prompt(cfg, 4), 8)
    assert checked >= 6


@pytest.mark.parametrize("name,ctxs", [
    ("smol135_w4", [0, 128]),   # tied bf16 head on int4 layers, 576-input rows
    ("llama7b_w4", [0, 2048]),
])
def test_w4a16_full_size(name, ctxs):
    cfg = si.get_config(name)
    pair = Pair(cfg)
    for ctx in ctxs:
        pair.dec.reset()
        pair.orc.reset()
        if ctx:
            pair.fill_kv(ctx)
        tok = si.make_prompt(cfg, 1, seed=10 + ctx)[0]
        g, am, ref, ref_am = pair.step(tok, ctx)
        compare(cfg, g, am, ref, ref_am, what=f"{name} ctx {ctx}")
    del pair
    torch.cuda.empty_cache()


def test_w4a16_greedy_32_steps():
    """The int4 path over many steps: SmolLM2 W4A16, 32 greedy steps."""
    cfg = si.get_config("smol135_w4")
    pair = Pair(cfg)
    worst, checked = greedy_teacher_forced(pair, si.make_prompt(cfg, 1), 31)
    assert checked >= 16
    del pair
    torch.cuda.empty_cache()


def test_tiny_device_token_chaining():
    """token_id = -1 feeds the previous step's device argmax (no host copy):
    the chained run must give exactly the tokens of a run whose tokens are
    read back and fed from the host (the kernel is deterministic)."""
    cfg = si.get_config("tiny")
    pair = Pair(cfg)
    prompt = si.make_prompt(cfg, 4)
    explicit = []
    tok = None
    for pos in range(12):
        tok = pair.dec.step(prompt[pos] if pos < 4 else tok, pos)
        if pos >= 3:
            explicit.append(tok)
    pair.dec.reset()
    for pos in range(4):
        first = pair.dec.step(prompt[pos], pos)
    chained = [first]
    for pos in range(4, 12):
        if pos < 11:
            pair.dec.step(-1, pos, want_argmax=False)
        else:
            chained.append(pair.dec.step(-1, pos))
    assert chained == [explicit[0], explicit[-1]]


def test_host_path_matches_device_path():
    cfg = si.get_config("tiny")
    pair = Pair(cfg)
    host = np.zeros(cfg.vocab, dtype=np.float32)
    a = pair.dec.step_host(5, 0, host)
    pair.dec.reset()
    b = pair.dec.step(5, 0, logits=pair.logits)
    assert a == b
    assert np.array_equal(host, pair.logits.cpu().numpy())


@pytest.mark.parametrize("name,ctxs", [
    ("smol135", [0, 128]),
    ("tinyllama", [0, 256, 1024]),
    ("llama1b_w8", [0, 512]),
    ("llama7b", [0, 2048]),
    ("llama7b_w8", [0, 2048]),
])
def test_full_size_single_steps(name, ctxs):
    cfg = si.get_config(name)
    pair = Pair(cfg)
    for ctx in ctxs:
        pair.dec.reset()
        pair.orc.reset()
        if ctx:
            pair.fill_kv(ctx)
        tok = si.make_prompt(cfg, 1, seed=10 + ctx)[0]
        g, am, ref, ref_am = pair.step(tok, ctx)
        compare(cfg, g, am, ref, ref_am, what=f"{name} ctx {ctx}")
    del pair
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name,ctx,fused", [
    ("tinyllama", 256, 2),     # the fused FFN level where the default keeps it split
    ("llama7b_w8", 0, 2),
    ("smol135", 128, 2),       # the fused level (level counters) where the default splits
    ("llama1b_w8", 512, 2),    # the fused int8 level (dp2a column loop), split by default
])
def test_ffn_level_variants(name, ctx, fused):
    """Both FFN schedules (one fused level with fixed-point accumulation of
    the down projection, or separate gate/up and down levels) against the
    oracle, on the shapes where the default picks the other one."""
    cfg = si.get_config(name)
    pair = Pair(cfg, options=amk.default_options(ffn_fused=fused))
    if ctx:
        pair.fill_kv(ctx)
    tok = si.make_prompt(cfg, 1, seed=10 + ctx)[0]
    g, am, ref, ref_am = pair.step(tok, ctx)
    compare(cfg, g, am, ref, ref_am, what=f"{name} ctx {ctx} ffn_fused {fused}")
    del pair
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name,ctx,stages,stage_bytes", [
    ("llama1b_w8", 512, 3, 65536),   # the bf16 ring shape on int8 weights
    ("tinyllama", 256, 4, 49152),    # the int8 ring shape on bf16 weights
    ("smol135", 128, 6, 32768),      # small stages: more chunks per task
    ("tinyllama", 0, 2, 98304),      # two large stages
])
def test_ring_shapes(name, ctx, stages, stage_bytes):
    """Ring shapes other than the weight format's default change the rows per
    chunk, the K split of the GEMV warps and the positions per attention
    chunk; every one must still match the oracle."""
    cfg = si.get_config(name)
    opts = amk.default_options(ring_stages=stages, stage_bytes=stage_bytes)
    pair = Pair(cfg, options=opts)
    st = pair.dec.stats()
    assert (st.ring_stages, st.stage_bytes) == (stages, stage_bytes)
    if ctx:
        pair.fill_kv(ctx)
    tok = si.make_prompt(cfg, 1, seed=10 + ctx)[0]
    g, am, ref, ref_am = pair.step(tok, ctx)
    compare(cfg, g, am, ref, ref_am, what=f"{name} ctx {ctx} ring {stages} x {stage_bytes}")
    del pair
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["tinyllama", "llama1b_w8", "tiny"])
def test_position0_schedule_matches_general(name):
    """At position 0 the schedule without the attention level gives the same
    logits, bit for bit, and the same KV-cache row 0 as the general one."""
    cfg = si.get_config(name)
    w = si.make_model(cfg, device="cuda")
    tok = si.make_prompt(cfg, 1, seed=10)[0]
    out = []
    for pos0 in (1, -1):
        dec = amk.Decoder(cfg, w, amk.default_options(pos0_plan=pos0))
        lg = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
        am = dec.step(tok, 0, logits=lg)
        kv0 = [torch.stack(dec.kv(l))[:, :, 0].clone() for l in range(cfg.n_layers)]
        out.append((lg.clone(), am, kv0))
        dec.close()
    assert torch.equal(out[0][0], out[1][0]) and out[0][1] == out[1][1]
    for a, b in zip(out[0][2], out[1][2]):
        assert torch.equal(a, b)


@pytest.mark.parametrize("edit", [
    dict(n_kv_heads=1),                 # one KV head for every query head (G = 4)
    dict(n_kv_heads=4),                 # plain multi-head attention (G = 1)
    dict(head_dim=128, n_heads=4, n_kv_heads=2, hidden=128),  # wide heads, G = 2
    dict(n_layers=3, ffn=256),          # FFN rows in 16-byte multiples: fused level
])
def test_tiny_shape_variants_to_the_last_cache_row(edit):
    """Greedy decode through every position of the cache (0 .. max_ctx - 1,
    the last row included) on variants of the tiny decoder, against the
    oracle, teacher-forced where the top-2 margin is within the bound."""
    cfg = si.get_config("tiny").with_(name="tiny_var", max_ctx=24, **edit)
    pair = Pair(cfg, options=amk.default_options(ffn_fused=2))
    prompt = si.make_prompt(cfg, 3)
    worst, checked = greedy_teacher_forced(pair, prompt, cfg.max_ctx - len(prompt))
    assert checked >= cfg.max_ctx // 2
    with pytest.raises(amk.AmkError) as e:
        pair.dec.step(1, cfg.max_ctx)
    assert e.value.name == "AMK_ERR_POS_RANGE"


@pytest.mark.parametrize("name", ["tinyllama", "llama1b_w8"])
def test_last_cache_row_full_size(name):
    """A full-size step at the last position the cache holds (max_ctx - 1,
    every earlier row filled): the longest split-K attention chunks and the
    last KV row, against the oracle."""
    cfg = si.get_config(name)
    pos = cfg.max_ctx - 1
    pair = Pair(cfg)
    pair.fill_kv(pos)
    tok = si.make_prompt(cfg, 1, seed=10)[0]
    g, am, ref, ref_am = pair.step(tok, pos)
    compare(cfg, g, am, ref, ref_am, f"{name} at the last cache row {pos}")
    del pair
    torch.cuda.empty_cache()


def test_ragged_sm_count_full_size():
    """A full-size shape on a prime number of CTAs (ragged tiles on every
    level, several tasks per queue) against the oracle at a long context."""
    cfg = si.get_config("tinyllama")
    pair = Pair(cfg, options=amk.default_options(n_sms=37))
    pair.fill_kv(300)
    tok = si.make_prompt(cfg, 1, seed=10)[0]
    g, am, ref, ref_am = pair.step(tok, 300)
    compare(cfg, g, am, ref, ref_am, "tinyllama on 37 CTAs, ctx 300")
    del pair
    torch.cuda.empty_cache()


def test_smol_greedy_32_steps():
    cfg = si.get_config("smol135")
    pair = Pair(cfg)
    worst, checked = greedy_teacher_forced(pair, si.make_prompt(cfg, 1), 31)
    assert checked >= 16


@pytest.mark.parametrize("name,prompt_len,n_new", [
    ("smol135", 128, 32),      # 32 greedy steps at KV context 128 (seeded 128-token prompt)
    ("tinyllama", 1, 32),      # 32 greedy steps from KV context 0
    ("llama1b_w8", 1, 32),     # the int8 path over many steps
])
def test_greedy_32_steps_full_size(name, prompt_len, n_new):
    """Greedy generation with the persistent KV cache at full size: the prompt
    is decoded through the real path (every step compared with the oracle),
    then n_new greedy steps, each token fed back; logits within the bound at
    every step and tokens exact wherever the oracle's top-2 margin exceeds
    it (teacher-forced past a near-tie)."""
    cfg = si.get_config(name)
    pair = Pair(cfg)
    prompt = si.make_prompt(cfg, prompt_len)
    worst, checked = greedy_teacher_forced(pair, prompt, n_new - 1)
    assert checked >= (prompt_len + n_new) // 2
    del pair
    torch.cuda.empty_cache()


def test_bad_arguments():
    cfg = si.get_config("tiny")
    pair = Pair(cfg)
    with pytest.raises(amk.AmkError) as e:
        pair.dec.step(0, cfg.max_ctx)
    assert e.value.name == "AMK_ERR_POS_RANGE"
    with pytest.raises(amk.AmkError) as e:
        pair.dec.step(cfg.vocab, 0)
    assert e.value.name == "AMK_ERR_POS_RANGE"
    with pytest.raises(amk.AmkError) as e:
        pair.dec.step(-1, 0)
    assert e.value.name == "AMK_ERR_INVALID_ARG"


@pytest.mark.parametrize("flagged", [1, -1])
def test_wait_timeout_is_reported_and_recoverable(flagged):
    """Fault injection on the host: one task never signals (level counters:
    its counter add is skipped; flagged waits: its flagged words carry a wrong
    tag), so a downstream wait runs out after its (short) limit; the kernel
    returns, the call reports AMK_ERR_TIMEOUT, the handle is poisoned until
    reset, and after a reset a normal handle decodes correctly again.  The
    general schedule runs at position 0 too, so that the attention level
    reads the victim's rows."""
    cfg = si.get_config("tiny")
    plan = amk.Plan(cfg, 4)
    kinds, _ = plan.task_info()
    victim = kinds.index(1)  # a QKV task
    opts = amk.default_options(n_sms=4, wait_timeout_us=20000, debug_skip_signal_task=victim,
                               flagged_waits=flagged, pos0_plan=-1)
    pair = Pair(cfg, options=opts)
    with pytest.raises(amk.AmkError) as e:
        pair.dec.step(3, 0)
    assert e.value.name == "AMK_ERR_TIMEOUT"
    info = pair.dec.error_info()
    assert info.code == 1 and info.task >= 0
    if flagged > 0:
        assert info.counter == -1  # a flagged read gave up: no counter
    else:
        assert info.counter >= 0
    with pytest.raises(amk.AmkError) as e:
        pair.dec.step(3, 0)
    assert e.value.name == "AMK_ERR_POISONED"
    pair.dec.reset()
    # the device context is still usable: a fresh handle on the same weights works
    good = Pair(cfg, weights=pair.w, options=amk.default_options(n_sms=4))
    g, am, ref, ref_am = good.step(3, 0)
    compare(cfg, g, am, ref, ref_am, "after timeout")


@pytest.mark.parametrize("name,ctx,steps,mode", [
    ("tiny", 0, 6, -1),
    ("tinyllama", 256, 2, -1),
    ("llama1b_w8", 512, 2, -1),
    ("llama7b", 0, 2, -1),
    ("smol135_w4", 0, 2, -1),
])
def test_wait_protocols_match_the_oracle(name, ctx, steps, mode):
    """The level-counter protocol (flagged_waits = -1) on models whose FFN
    levels are split, where flagged waits are the default: the same logits
    within the tolerance, steps chained on the device."""
    cfg = si.get_config(name)
    pair = Pair(cfg, options=amk.default_options(flagged_waits=mode))
    if ctx:
        pair.fill_kv(ctx)
    prompt = si.make_prompt(cfg, steps)
    for i, t in enumerate(prompt):
        g, am, ref, ref_am = pair.step(t, ctx + i)
        compare(cfg, g, am, ref, ref_am, what=f"{name} waits {mode} pos {ctx + i}")
    del pair
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name,ctx,steps", [
    ("tiny", 0, 12),          # split FFN levels, attention at every position up to 11
    ("smol135", 120, 6),      # fused FFN level, several split-K attention chunks
    ("llama1b_w8", 500, 3),   # int8, long cache
])
def test_debug_checks_keep_every_buffer_in_bounds(name, ctx, steps):
    """With debug checks on, amk_create bounds-checks every task record, and
    after several steps (parity-checked) no kernel or copy has written into
    the guard after any of the handle's device buffers."""
    cfg = si.get_config(name)
    pair = Pair(cfg, options=amk.default_options(debug_checks=1))
    if ctx:
        pair.fill_kv(ctx)
    prompt = si.make_prompt(cfg, steps)
    for i, t in enumerate(prompt):
        g, am, ref, ref_am = pair.step(t, ctx + i)
        compare(cfg, g, am, ref, ref_am, what=f"{name} debug pos {ctx + i}")
    assert pair.dec.check_guards() == 0
    del pair
    torch.cuda.empty_cache()
