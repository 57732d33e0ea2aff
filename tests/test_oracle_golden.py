"""The oracle against the hand-derived example in tests/golden/ (no GPU)."""
import json
import os

import numpy as np

from sparse_attention_indexer_head_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example_d4.json")


def _bf(x):
    return W.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _f(bits):
    return W.bf16_bits_to_f32(bits)


def test_worked_example(orc):
    g = json.load(open(GOLDEN))
    i, e = g["inputs"], g["expected"]
    kp, P = i["kpool"], i["max_pools"]
    keys, idx, pv, fv = orc.kpool_compress(
        _bf(i["k"]), _bf(i["gate"]), np.asarray(i["valid"], np.uint8),
        np.asarray(i["req_start"], np.int32), kp, P, np.asarray(i["ape"], np.float32),
        _bf(i["ln_w"]), _bf(i["ln_b"]), i["eps"])
    assert fv.tolist() == e["first_valid"]
    assert pv.tolist() == e["pool_valid"]
    assert idx.tolist() == e["pool_idx"]
    np.testing.assert_array_equal(_f(keys[:, :2]), np.asarray(e["pool_keys_valid_rows"], np.float32))

    scores, cand = orc.index_scores(_bf(i["q_idx"]), np.asarray(i["gate_w"], np.float32),
                                    np.asarray(i["q_req"], np.int32),
                                    np.asarray(i["q_pos"], np.int32), keys, pv, fv, kp)
    assert cand.tolist() == e["cand"]
    np.testing.assert_array_equal(scores, np.asarray(e["scores"], dtype=np.float32))

    top, ids = orc.topk_expand(scores, cand, idx, np.asarray(i["q_req"], np.int32), i["select_k"])
    assert top.tolist() == e["top_pools"]
    assert ids.tolist() == e["token_ids"]

    out, lse = orc.sparse_mla(_bf(i["q_mla"]), _bf(i["kv"]), np.asarray(i["req_start"], np.int32),
                              np.asarray(i["q_req"], np.int32), ids, i["sm_scale"])
    np.testing.assert_array_equal(_f(out), np.asarray(e["out"], np.float32))
    np.testing.assert_allclose(lse, np.asarray(e["lse"], np.float32), rtol=1e-7)
