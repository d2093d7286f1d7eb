"""The oracle still reproduces its stored outputs for the tiny fp32 workload
(tests/golden/cfg1_oracle.json, written by tests/golden/make_golden.py from the oracle only)."""
import json
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_matches_stored_golden():
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_golden",
                                                  os.path.join(HERE, "golden", "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    with open(os.path.join(HERE, "golden", "cfg1_oracle.json")) as f:
        stored = json.load(f)
    now = mg.compute()
    assert stored.keys() == now.keys()
    for k in stored:
        for name, v in stored[k].items():
            np.testing.assert_allclose(np.asarray(now[k][name]), np.asarray(v), rtol=1e-12,
                                       atol=1e-15, err_msg=f"{k} {name}")
