"""The decode loop's schedule and byte count, built on the CPU (no kernel runs):
123 boundaries for 61 layers in the order of the layer loop, the captured
layers, and the algorithmic bytes of each kind of boundary."""

from mhc_residual_stream_b200 import build
from mhc_residual_stream_b200.decode import DecodeLoop


def _loop(layers=61, rows=4, **kw):
    build.build()
    return DecodeLoop(rows=rows, layers=layers, device="cpu", pack_fn=False, **kw)


def test_schedule_order_and_slots():
    loop = _loop()
    kinds = [st.kind for st in loop.steps]
    assert len(kinds) == 123
    assert kinds[0] == "first" and kinds[1] == "ffn" and kinds[-1] == "final"
    assert kinds[1:-1] == ["ffn"] + ["attn", "ffn"] * 60
    # attention entries finalize the previous MoE and quantize; FFN entries sum partials
    for st in loop.steps[1:-1]:
        assert (st.pending.kind == "moe") == (st.kind == "attn") == st.mxfp8
    assert loop.steps[-1].pending.kind == "moe"
    # the state ping-pongs: every boundary reads the slot the previous one wrote
    for a, b in zip(loop.steps, loop.steps[1:]):
        assert b.src == a.dst and b.dst == 1 - b.src
    assert loop.final_slot == loop.steps[-1].dst


def test_captured_layers():
    loop = _loop()
    assert loop.aux_layers == (2, 30, 58, 61)
    captured = [(st.kind, st.layer) for st in loop.steps if loop.aux_of(st) is not None]
    assert captured == [("attn", 2), ("attn", 30), ("attn", 58), ("final", 61)]
    assert tuple(_loop(layers=3, aux_layers=()).aux) == ()


def test_algorithmic_bytes_by_kind():
    R, H, n, P, k = 4, 7168, 4, 8, 8
    C = 2 * n + n * n
    loop = _loop(rows=R, layers=3, aux_layers=())
    fn_b = n * H * C * 4 + (3 + C) * 4
    mix = R * C * 4
    first = R * H * 2 + R * n * H * 2 + R * H * 2 + fn_b + H * 2 + mix
    ffn = P * R * H * 2 + 2 * R * n * H * 2 + mix + R * H * 2 + H * 2 + fn_b + mix
    scales = ((R + 127) // 128 * 128) * ((H // 32 + 3) // 4 * 4)
    moe_in = (R * k + R) * H * 2 + R * k * 8
    attn = moe_in + 2 * R * n * H * 2 + mix + R * H * 2 + H * 2 + fn_b + mix + R * H + scales
    final = moe_in + 2 * R * n * H * 2 + mix + R * H * 2 + H * 2
    assert loop.algorithmic_bytes() == first + ffn + 2 * (attn + ffn) + final
    with_aux = _loop(rows=R, layers=3, aux_layers=(2, 3))
    assert with_aux.algorithmic_bytes() == loop.algorithmic_bytes() + 2 * R * H * 2


def test_engram_layers_split_the_attention_entry():
    loop = _loop(layers=6, engram_layers=(2, 4), aux_layers=(2, 3))
    kinds = [(st.kind, st.layer) for st in loop.steps]
    assert kinds == [("first", 0), ("ffn", 0), ("attn", 1), ("ffn", 1), ("post_only", 2), ("engram", 2), ("ffn", 2),
                     ("attn", 3), ("ffn", 3), ("post_only", 4), ("engram", 4), ("ffn", 4), ("attn", 5), ("ffn", 5),
                     ("final", 6)]
    # the finalize and the injected streams' coefficients share the slot pair of one boundary
    po, en = loop.steps[4], loop.steps[5]
    assert (po.src, po.dst) == (en.src, en.dst)
    for a, b in zip(loop.steps, loop.steps[1:]):
        if b.kind != "engram":
            assert b.src == a.dst
    # an Engram layer captures the streams before the injection
    assert loop.aux_of(po) is loop.aux[2] and loop.aux_of(en) is None
    R, H, n = 4, 7168, 4
    C = 2 * n + n * n
    fn_b = n * H * C * 4 + (3 + C) * 4
    plain = _loop(layers=6, aux_layers=())
    eng = _loop(layers=6, engram_layers=(2,), aux_layers=())
    attn2 = [st for st in plain.steps if st.kind == "attn" and st.layer == 2][0]
    scales = ((R + 127) // 128 * 128) * ((H // 32 + 3) // 4 * 4)
    moe_in = (R * 8 + R) * H * 2 + R * 8 * 8
    attn_b = moe_in + 2 * R * n * H * 2 + R * C * 4 + R * H * 2 + H * 2 + fn_b + R * C * 4 + R * H + scales
    split_b = (moe_in + 2 * R * n * H * 2 + R * (n + n * n) * 4) + (R * n * H * 2 + R * n * 4 + fn_b + H * 2
                                                                     + R * H * 2 + R * C * 4)
    assert attn2.mxfp8
    assert eng.algorithmic_bytes() - plain.algorithmic_bytes() == split_b - attn_b
