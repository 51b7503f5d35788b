"""Host lowering: every workload lowers to a schedule the validator accepts,
its tiles cover each weight matrix exactly once, and a small real lowering
also passes the brute-force interleaving checker.

paperfeed "RightNow-AI/AutoMegaKernel", "How it works": model -> tiled task
DAG; x-techcon AutoMegaKernel article, section 1: all real lowerings accepted.
"""
import pytest

import persistent_megakernel_decode_cta_b200 as amk
from persistent_megakernel_decode_cta_b200 import abi, build
import synth_inputs as si
from oracle import interleave as bf

KIND = {1: "QKV", 2: "ATTN", 3: "OPROJ", 4: "GATEUP", 5: "DOWN", 6: "LMHEAD", 7: "FFN"}
ORDER = ["QKV", "ATTN", "OPROJ", "GATEUP", "DOWN", "FFN", "LMHEAD"]


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def _writes(g, buf, kind=None):
    out = []
    for t, task in enumerate(g["tasks"]):
        for (b, k, lo, hi) in task["accesses"]:
            if b == buf and k == (abi.ACC_WRITE if kind is None else kind):
                out.append((lo, hi, t))
    return sorted(out)


def _partition(ranges, size):
    pos = 0
    for lo, hi, _ in ranges:
        assert lo == pos, (lo, pos)
        pos = hi
    assert pos == size


@pytest.mark.parametrize("name", list(si.CONFIGS))
@pytest.mark.parametrize("n_sms", [148, 7])
@pytest.mark.parametrize("fused", [2, -1])
def test_real_lowerings_accepted_and_cover(name, n_sms, fused):
    cfg = si.get_config(name)
    plan = amk.Plan(cfg, n_sms, amk.default_options(ffn_fused=fused))
    g = plan.graph()
    kinds, layers = plan.task_info()
    L, h, F = cfg.n_layers, cfg.hidden, cfg.ffn
    is_fused = any(KIND[k] == "FFN" for k in kinds)
    if fused < 0:
        assert not is_fused
    # buffers: 6 per layer (qkv, attention output, xmid, xout, act, kvnew) +
    # logits, key, key_next
    assert len(g["buffers"]) == 6 * L + 3
    for l in range(L):
        _partition(_writes(g, 6 * l + 0), cfg.q_rows + 2 * cfg.kv_rows)   # QKV rows
        _partition(_writes(g, 6 * l + 2), h)                               # O rows
        # down rows, or (fused) the O rows that start the FFN's accumulator
        _partition(_writes(g, 6 * l + 3), h)
        if is_fused:
            acc = _writes(g, 6 * l + 3, abi.ACC_ACCUM)
            ffn = [t for t in range(len(kinds)) if KIND[kinds[t]] == "FFN" and layers[t] == l]
            assert sorted(t for _, _, t in acc) == ffn
            assert all((lo, hi) == (0, h) for lo, hi, _ in acc)
        else:
            _partition(_writes(g, 6 * l + 4), F)                           # gate/up rows
    _partition(_writes(g, 6 * L), cfg.vocab)                               # LM head rows
    # every SM runs its tasks level by level
    for q in g["queues"]:
        seq = [(layers[t], ORDER.index(KIND[kinds[t]])) for t in q]
        assert seq == sorted(seq)
    n_att = sum(1 for k in kinds if KIND[k] == "ATTN")
    assert n_att % (L * cfg.n_kv_heads) == 0
    # the library's validator accepts the plan (it ran inside amk_plan_create
    # too); run it again on the exported graph
    ok, rule, msg = amk.validate_graph(g)
    assert ok, (rule, msg)


@pytest.mark.parametrize("name", list(si.CONFIGS))
@pytest.mark.parametrize("fused", [2, -1])
def test_position0_schedule(name, fused):
    """The position-0 schedule has no attention level; its O-projection reads
    the K/V rows, the O tiles write KV row 0 in shares that tile it, and the
    validator accepts it."""
    cfg = si.get_config(name)
    plan = amk.Plan(cfg, 148, amk.default_options(ffn_fused=fused))
    z = plan.pos0()
    assert z is not None
    g = z.graph()
    kinds, layers = z.task_info()
    assert not any(KIND[k] == "ATTN" for k in kinds)
    L, nh, nkv, hd = cfg.n_layers, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    for l in range(L):
        kvnew = _writes(g, 6 * l + 5)
        _partition(kvnew, 2 * nkv * hd)
        assert all(KIND[kinds[t]] == "OPROJ" for _, _, t in kvnew)
    for q in g["queues"]:
        seq = [(layers[t], ORDER.index(KIND[kinds[t]])) for t in q]
        assert seq == sorted(seq)
    ok, rule, msg = amk.validate_graph(g)
    assert ok, (rule, msg)
    assert amk.Plan(cfg, 148, amk.default_options(pos0_plan=-1)).pos0() is None


def test_fused_ffn_slices_cover_ffn():
    """The fused FFN level of each layer has about one slice per SM, each a
    multiple of 16 bytes of a Wdown row, and the slices tile [0, ffn)."""
    for name in ("tinyllama", "llama1b_w8", "llama7b", "smol135"):
        cfg = si.get_config(name)
        plan = amk.Plan(cfg, 148, amk.default_options(ffn_fused=2))
        kinds, layers = plan.task_info()
        n = sum(1 for k, l in zip(kinds, layers) if KIND[k] == "FFN" and l == 0)
        esz = 1 if cfg.quant == "w8a16" else 2
        w = -(-(cfg.ffn // (16 // esz)) // 148) * (16 // esz)
        assert n == -(-cfg.ffn // w) and n <= 148, (name, n)


@pytest.mark.parametrize("flagged", [1, -1])
@pytest.mark.parametrize("pos0", [False, True])
def test_small_real_lowering_passes_brute_force(flagged, pos0):
    """Every interleaving of a one-layer lowering is safe, with the waits on
    the flagged words (default) or on the level counters, and for the
    general schedule as for the position-0 one (no attention level)."""
    cfg = si.get_config("tiny").with_(n_layers=1, name="tiny1")
    opts = amk.default_options(attn_splits=1, flagged_waits=flagged)
    plan = amk.Plan(cfg, 2, opts)
    assert plan.stats().flagged_waits == (1 if flagged > 0 else 0)
    g = (plan.pos0() if pos0 else plan).graph()
    assert len(g["tasks"]) <= 14
    assert bf.check(g) == (True, "ok")


def test_balanced_tiles_on_148_sms():
    cfg = si.get_config("tinyllama")
    plan = amk.Plan(cfg, 148, amk.default_options(ffn_fused=-1))
    g = plan.graph()
    kinds, layers = plan.task_info()
    per_sm_gateup = [sum(1 for t in q if kinds[t] == 4 and layers[t] == 0) for q in g["queues"]]
    assert max(per_sm_gateup) == 1 and min(per_sm_gateup) == 1
    fused = amk.Plan(cfg, 148, amk.default_options(ffn_fused=2))
    g = fused.graph()
    kinds, layers = fused.task_info()
    per_sm_ffn = [sum(1 for t in q if kinds[t] == 7 and layers[t] == 0) for q in g["queues"]]
    assert max(per_sm_ffn) == 1


@pytest.mark.parametrize("edit,status", [
    (dict(head_dim=12), "AMK_ERR_UNSUPPORTED"),          # KV rows not 16-byte multiples
    (dict(n_kv_heads=3), "AMK_ERR_UNSUPPORTED"),         # 4 heads not divisible by 3
    (dict(ffn=12290), "AMK_ERR_UNSUPPORTED"),            # down K above the register slice
    (dict(hidden=0), "AMK_ERR_INVALID_ARG"),
    (dict(ffn=171), "AMK_ERR_UNSUPPORTED"),              # odd bf16 K: row not 4-byte aligned
    (dict(quant="w4a16"), "AMK_ERR_UNSUPPORTED"),        # int4 rows of 172 inputs: not 32-multiples
])
def test_unsupported_shapes_rejected(edit, status):
    cfg = si.get_config("tiny").with_(**edit)
    with pytest.raises(amk.AmkError) as e:
        amk.Plan(cfg, 4)
    assert e.value.name == status


def test_bad_options_rejected():
    cfg = si.get_config("tiny")
    with pytest.raises(amk.AmkError) as e:
        amk.Plan(cfg, 4, amk.default_options(stage_bytes=1000))
    assert e.value.name == "AMK_ERR_INVALID_ARG"


@pytest.mark.parametrize("name", ["tiny", "smol135", "tinyllama", "llama1b_w8", "llama7b",
                                  "llama7b_w8"])
def test_ring_shape_resolved_per_weight_format(name):
    """Left at 0, the ring takes 48 KiB stages for int8 weights and 64 KiB for
    bf16, as many as make 192 KiB; explicit values are kept."""
    cfg = si.get_config(name)
    st = amk.Plan(cfg, 148).stats()
    want = (4, 48 * 1024) if cfg.quant == "w8a16" else (3, 64 * 1024)
    assert (st.ring_stages, st.stage_bytes) == want
    assert st.n_tasks > 0 and st.epoch == 0 and st.smem_bytes <= 227 * 1024
    st = amk.Plan(cfg, 148, amk.default_options(stage_bytes=32768)).stats()
    assert (st.ring_stages, st.stage_bytes) == (6, 32768)
    st = amk.Plan(cfg, 148, amk.default_options(ring_stages=2, stage_bytes=65536)).stats()
    assert (st.ring_stages, st.stage_bytes) == (2, 65536)


@pytest.mark.parametrize("name", ["smol135_w4", "llama7b_w4", "tinyllama", "llama1b_w8"])
def test_w4a16_lowering(name):
    """int4 plans: 48 KiB stages, split FFN levels, and streamed bytes equal
    to the codes and group scales plus the padding of each row to 16 bytes."""
    cfg = si.get_config(name).with_(quant="w4a16")
    st = amk.Plan(cfg, 148).stats()
    assert (st.ring_stages, st.stage_bytes) == (4, 48 * 1024)
    sb = si.streamed_weight_bytes(cfg)
    assert sb <= st.weight_bytes <= sb * 1.025
    kinds, _ = amk.Plan(cfg, 148, amk.default_options(ffn_fused=2)).task_info()
    assert 7 not in kinds  # no fused FFN level for int4 weights


def test_w4a16_rows_need_whole_code_vectors():
    cfg = si.get_config("tiny").with_(quant="w4a16", ffn=192)
    amk.Plan(cfg, 4)
    with pytest.raises(amk.AmkError) as e:
        amk.Plan(cfg.with_(ffn=176), 4)
    assert e.value.name == "AMK_ERR_UNSUPPORTED"


def test_noalloc_refuses_int4_models_on_the_host():
    """int4 weights are packed by amk_create, which allocates: the
    no-allocation step refuses them before any device work (the pointers
    below are aligned stand-ins that are never dereferenced)."""
    import ctypes
    from persistent_megakernel_decode_cta_b200 import abi
    cfg = si.get_config("smol135_w4")
    plan = amk.Plan(cfg, 148)
    fake = 1 << 20
    ptrs = (ctypes.c_void_p * cfg.n_layers)(*([fake] * cfg.n_layers))
    ws = abi.Weights()
    for f in ("embed", "final_norm"):
        setattr(ws, f, fake)
    for name in ("attn_norm", "ffn_norm", "wq", "wk", "wv", "wo", "wgate", "wup", "wdown",
                 "sq", "sk", "sv", "so", "sgate", "sup", "sdown"):
        setattr(ws, name, ctypes.cast(ptrs, abi.c_vpp))
    lib = abi.lib()
    rc = lib.amk_decode_step_noalloc(plan._p, ctypes.byref(ws), fake, 0, 0, fake, None, None)
    assert rc == abi.ERR["AMK_ERR_UNSUPPORTED"]
    assert b"int4" in lib.amk_last_error()
    plan.close()


def test_sm_rotation_moves_tiles_not_balance():
    """The SM-assignment knob: a rotated plan validates, keeps every level's
    bytes per SM as balanced as the default plan, and puts tiles on other SMs."""
    cfg = si.get_config("tinyllama")
    a = amk.Plan(cfg, 148)
    b = amk.Plan(cfg, 148, amk.default_options(sm_rotate=37))
    ga, gb = a.graph(), b.graph()
    assert len(ga["tasks"]) == len(gb["tasks"])
    sa = [t["sm"] for t in ga["tasks"]]
    sb = [t["sm"] for t in gb["tasks"]]
    # levels with fewer tiles than SMs leave other SMs idle under rotation, so
    # queue lengths move a little; the tiles and their bytes do not change
    la = [len(q) for q in ga["queues"]]
    lb = [len(q) for q in gb["queues"]]
    assert max(lb) - min(lb) <= max(la) - min(la) + 3
    ka, _ = a.task_info()
    kb, _ = b.task_info()
    assert sorted(ka) == sorted(kb)
    assert sa != sb
    assert a.stats().weight_bytes == b.stats().weight_bytes


@pytest.mark.parametrize("name,fused_with_counters", [
    ("tinyllama", 0), ("llama7b", 0), ("llama1b_w8", 0), ("llama7b_w8", 0),
    ("smol135", 1),  # residual rows of 1152 B: fused when the counters are asked for
])
def test_flagged_waits_resolution(name, fused_with_counters):
    """Flagged waits with separate FFN levels are the default everywhere; with
    flagged_waits = -1 the level counters come back, and with them the fused
    FFN level on narrow residuals; a fused level (forced) always runs on the
    counters (its residual is a fixed-point sum)."""
    cfg = si.get_config(name)
    st = amk.Plan(cfg, 148).stats()
    assert (st.flagged_waits, st.ffn_fused) == (1, 0)
    off = amk.Plan(cfg, 148, amk.default_options(flagged_waits=-1)).stats()
    assert (off.flagged_waits, off.ffn_fused) == (0, fused_with_counters)
    fused = amk.Plan(cfg, 148, amk.default_options(ffn_fused=2)).stats()
    if fused.ffn_fused:
        assert fused.flagged_waits == 0
