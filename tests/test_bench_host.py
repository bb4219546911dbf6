"""Host-side logic of bench.py that needs no GPU: the digest that ties the committed DRAM
traffic record to the decode kernel's code, and the record's own arithmetic."""
import json
import os

import bench
from tests.conftest import ROOT


def test_code_digest_ignores_comments_and_layout_but_not_code():
    src = 'int f(int a) {\n  // add one\n  return a + 1; /* done */\n}\nconst char *s = "x // y";\n'
    reflowed = 'int f(int a)\n{\n    /* adds\n       one */ return a + 1;\n}\nconst char *s = "x // y"; // note\n'
    assert bench._code_only(src) == bench._code_only(reflowed)
    assert bench._code_only(src) != bench._code_only(src.replace("a + 1", "a + 2"))
    # text inside string literals is code, not a comment
    assert bench._code_only(src) != bench._code_only(src.replace('"x // y"', '"x"'))


def test_traffic_record_is_consistent():
    with open(os.path.join(ROOT, "profiles", "decode_traffic.json")) as f:
        rec = json.load(f)
    # the bench launch processes twice the captured units: reads double, partial writes do not
    assert rec["dram_bytes_per_launch"] == 2 * rec["dram_read_bytes_captured"] + rec["dram_write_bytes_captured"]
    assert rec["captured_T"] * 2 == 32768
    assert len(rec["sources_sha256"]) == 64
    # the captured DRAM reads are within 1% of the packed bytes of the captured launch
    packed = 16 * 8 * rec["captured_T"] * (66 + 34)
    assert abs(rec["dram_read_bytes_captured"] - packed) < 0.01 * packed


def test_boundary_flip_count_of_the_oracle_leg():
    # device codes equal to the oracle's give no flips; one code changed away from a decision
    # boundary is counted as such
    import numpy as np

    import oracle as O
    from quantized_decode_attention_kv_b200.workloads import WORKLOADS
    w = WORKLOADS["llama3_8b_decode_32k"]
    rng = np.random.default_rng(0)
    kx = rng.standard_normal((64, 128))
    vx = rng.standard_normal((64, 128))
    kr = O.quantize(kx, w.k_bits, seed=w.seed)
    vr = O.quantize(vx, w.v_bits, seed=w.seed)
    kcodes, vcodes = kr.packed.copy(), vr.packed.copy()
    res = bench.oracle_boundary_flips(w, 64, kx, kcodes, None, vx, vcodes, None)
    assert res["k"]["flipped"] == 0 and res["v"]["flipped"] == 0
    assert res["k"]["coords"] == 64 * 128
    far = np.argmax(O.boundary_distance(kr)[3])
    codes = kr.codes.copy()
    codes[3, far] ^= 1
    res = bench.oracle_boundary_flips(w, 64, kx, O.pack_bits(codes, w.k_bits), None, vx, vcodes, None)
    assert res["k"]["flipped"] == 1 and res["k"]["flipped_away_from_boundary"] == 1
