"""Writes tiny_oracle.json: the oracle's own greedy decode of the seeded tiny
workload (prompt prefilled by full causal recompute, then 8 greedy steps), as a
regression record of the oracle.

The pages print no decoded sequence, logit or hidden state for any model, so
these values are not pins of the oracle to the pages (its pins are in
test_oracle_pins.py); they record what the oracle computes today, so that a
change to its arithmetic shows up as a failing test_golden.py and has to be
justified.  Only oracle/ and the seeded generators (synth/) are called.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import torch  # noqa: E402

import synth  # noqa: E402
from oracle import OracleDecoder  # noqa: E402

STEPS = 8


def compute():
    cfg = synth.get_config("tiny")
    w = synth.make_weights(cfg, norm_std=0.1)
    prompt = synth.make_prompt(cfg)                      # [1][kv_len + 1]
    o = OracleDecoder(cfg, w, 1, max_seq=cfg.kv_len + STEPS + 1)
    o.forward_sequence(prompt[:, : cfg.kv_len])
    tok = int(prompt[0, cfg.kv_len])
    steps = []
    for _ in range(STEPS):
        logits, hidden = o.step([tok])
        top = torch.topk(logits[0], 5)
        steps.append({"input": tok,
                      "top5_index": [int(i) for i in top.indices],
                      "top5_logit": [float(v) for v in top.values],
                      "logit_l2": float(logits[0].double().norm()),
                      "hidden_l2": float(hidden[0].double().norm())})
        tok = int(top.indices[0])
    return {"workload": "tiny (seeded), gains 1 + N(0, 0.1^2), prompt prefilled, greedy", "steps": steps}


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_oracle.json"), "w") as f:
        json.dump(compute(), f, indent=1)
        f.write("\n")
