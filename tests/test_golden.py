"""The oracle against its recorded decode of the tiny workload
(tests/golden/tiny_oracle.json, written by tests/golden/make_golden.py from the
oracle alone).  A failure means the oracle's arithmetic changed: the change has
to be justified by the pages, and the record rewritten.  CPU only."""
import json
import os

import pytest

from tests.golden.make_golden import compute

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_oracle_matches_its_record():
    rec = json.load(open(os.path.join(HERE, "tiny_oracle.json")))
    now = compute()
    assert len(now["steps"]) == len(rec["steps"])
    for s, (a, b) in enumerate(zip(now["steps"], rec["steps"])):
        assert a["input"] == b["input"], s
        assert a["top5_index"] == b["top5_index"], s
        assert a["top5_logit"] == pytest.approx(b["top5_logit"], rel=1e-5, abs=1e-5), s
        assert a["logit_l2"] == pytest.approx(b["logit_l2"], rel=1e-5), s
        assert a["hidden_l2"] == pytest.approx(b["hidden_l2"], rel=1e-5), s
