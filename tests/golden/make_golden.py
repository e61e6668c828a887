"""Write tests/golden/tiny_step_oracle.json from the fp64 oracle (and nothing else).

The pages print no worked numbers for the decode math, so this fixture is not a page
value: it is a regression record of the pinned oracle on the tiny 2-layer workload
(hidden 256, 4 q / 2 kv heads of dim 64, SwiGLU 688, vocab 1024, 128 cached positions),
one decode step at pos 128 from the workload's seed-fixed token.  Re-run only when a
commit that changes the oracle's arithmetic names the passage that justifies it.
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from persistent_tile_pipelined_b200.synth import workloads as W  # noqa: E402


def main():
    wl = W.TINY
    m = W.gen_gqa_model(wl)
    tok = W.first_token(wl)
    logits, hidden = oracle.Oracle(64).decode_step(wl, m, tok, wl.prefill)
    rec = {
        "workload": wl.name, "seed": wl.seed, "token": tok, "pos": wl.prefill,
        "argmax": int(np.argmax(logits)),
        "logits_head": [float(v) for v in logits[:32]],
        "logits_l2": float(np.linalg.norm(logits)),
        "hidden_l2": [float(np.linalg.norm(h)) for h in hidden],
        "k_cache_row": [int(v) for v in m["k_cache"][1][1, wl.prefill, :16]],
    }
    with open(os.path.join(HERE, "tiny_step_oracle.json"), "w") as f:
        json.dump(rec, f, indent=1)
    print(json.dumps(rec)[:200])


if __name__ == "__main__":
    main()
