"""The oracle still reproduces its recorded output on the tiny workload (regression)."""
import json
import os

import numpy as np

import oracle
from persistent_tile_pipelined_b200.synth import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))


def test_tiny_step_matches_record():
    rec = json.load(open(os.path.join(HERE, "golden", "tiny_step_oracle.json")))
    wl = W.TINY
    assert rec["workload"] == wl.name and rec["seed"] == wl.seed
    m = W.gen_gqa_model(wl)
    assert W.first_token(wl) == rec["token"]
    logits, hidden = oracle.Oracle(64).decode_step(wl, m, rec["token"], rec["pos"])
    np.testing.assert_allclose(logits[:32], rec["logits_head"], rtol=1e-12, atol=1e-12)
    assert int(np.argmax(logits)) == rec["argmax"]
    np.testing.assert_allclose(np.linalg.norm(logits), rec["logits_l2"], rtol=1e-12)
    np.testing.assert_allclose([np.linalg.norm(h) for h in hidden], rec["hidden_l2"], rtol=1e-12)
    assert [int(v) for v in m["k_cache"][1][1, rec["pos"], :16]] == rec["k_cache_row"]
