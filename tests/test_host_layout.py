"""Host logic that needs no GPU: the staging layout of TreeVerifier's end-to-end
path and the benchmark's choice of roofline bound."""
import torch

import bench
from tree_speculative_decoding_04_b200.verifier import _InputLayout


def _ranges(lay):
    out = [("meta", 0, lay.meta_bytes), ("logits", lay.logits_off, lay.logits_off + lay.logits_bytes)]
    for layer in range(lay.L):
        o = lay.layer_off(layer)
        out.append((f"layer{layer}", o, o + lay.q_bytes + 2 * lay.rows_bytes))
    return out


def test_sections_are_aligned_disjoint_and_inside_the_buffer():
    for shape in [(1, 17, 4, 4, 64, 1024, 1), (1, 65, 32, 32, 128, 32000, 32), (8, 6, 32, 8, 128, 151936, 3),
                  (32, 17, 32, 2, 128, 151552, 2), (3, 1, 2, 1, 64, 7, 5)]:
        lay = _InputLayout(*shape)
        rs = sorted(_ranges(lay), key=lambda r: r[1])
        for (_, a0, a1), (_, b0, _) in zip(rs, rs[1:]):
            assert a1 <= b0
        assert rs[-1][2] <= lay.nbytes and lay.nbytes % 256 == 0
        for name, a0, _ in rs:
            assert a0 % 256 == 0 or name == "meta"


def test_views_are_contiguous_per_layer_and_land_in_their_sections():
    lay = _InputLayout(3, 7, 8, 2, 128, 1000, 4)
    buf = torch.zeros(lay.nbytes, dtype=torch.uint8)
    v = lay.views(buf)
    assert v["parent"].shape == (3, 7) and v["logits"].shape == (3, 7, 1000)
    for layer in range(lay.L):
        for key in ("q", "tree_k", "tree_v"):
            assert v[key][layer].is_contiguous()
    # each view writes exactly its own bytes
    marks = {"parent": 1, "draft": 2, "logits": 3}
    for key, val in marks.items():
        v[key].fill_(val)
    v["tree_v"][2].fill_(1.0)
    b = buf.numpy()
    assert (b[:lay.draft_off].view("int32") == 1).all()
    assert (b[lay.draft_off:lay.meta_bytes].view("int32") == 2).all()
    assert (b[lay.logits_off:lay.logits_off + lay.logits_bytes].view("float32") == 3).all()
    o = lay.layer_off(2) + lay.q_bytes + lay.rows_bytes
    assert (buf[o:o + lay.rows_bytes].view(torch.bfloat16) == 1.0).all()
    assert int(buf[lay.layers_off:o].sum()) == 0 and int(buf[o + lay.rows_bytes:].sum()) == 0


def test_roofline_bound_is_the_larger_term():
    hbm, tf = 6550.4, 1403.3
    # mha7b-like: 35.7 MB and 2.2 GFLOP per launch -> bandwidth-bound
    r = bench.roofline_entry(35_684_352, 2.19e9, 15.7e-3, hbm, tf, "measured", None, "k")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["achieved"] - 35_684_352 / 15.7e-6 / 1e9) < 1e-6 and abs(r["frac"] - r["achieved"] / hbm) < 1e-12
    # b32gqa-like: 278 MB and 73 GFLOP per launch -> tensor-bound at the sustained peak
    r = bench.roofline_entry(278e6, 73e9, 153e-3, hbm, tf, "measured", 290e6, "k")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] == tf and r["traffic"] == 290e6
    assert abs(r["frac"] - 73e9 / 153e-6 / 1e12 / tf) < 1e-12
