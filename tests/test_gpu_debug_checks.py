"""LSA_DEBUG=1: the library's checks at the ABI boundary.

A child process (tests/debug_child.py) loads the library with LSA_DEBUG=1.
The same small pipeline (tests/debug_case.py: index build, a prefill chunk,
a selection, a per-key selection, a sparse attention) passes every check and
gives the results it gives without them (run here, in this process): the
same selections, the same attention within bf16 rounding.
Three corruptions planted from the host between calls are refused with
LSA_ERR_INTERNAL before any kernel reads them: a gather index past T_cap, a
chunk selection with a long-range key after its query, and two bucket members
swapped in the index's CSR.
"""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

lsa = pytest.importorskip("long_context_indexing_b200")

HERE = os.path.dirname(os.path.abspath(__file__))


def test_debug_checks_pass_clean_runs_and_refuse_corruption(tmp_path):
    out_json, out_pt = str(tmp_path / "found.json"), str(tmp_path / "clean.pt")
    env = dict(os.environ, LSA_DEBUG="1")
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_child.py"), out_json, out_pt],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    found = json.load(open(out_json))
    assert found["clean"] is True
    for what, words in (("gather", "outside [0, T_cap)"), ("selection", "after its query"),
                        ("index", "not ascending")):
        f = found[what]
        assert f is not None, what
        assert f["code"] == 6 and "debug check" in f["msg"] and words in f["msg"], (what, f)
    # the checked run's outputs equal an unchecked run's
    sys.path.insert(0, HERE)
    from debug_case import case
    _, _, _, _, res = case(lsa)
    ref = torch.load(out_pt)
    for k, v in res.items():
        if v.dtype == torch.int32:
            assert torch.equal(v.cpu(), ref[k]), k
        else:                       # attention: the bucket path's plan order comes from atomics
            assert (v.cpu().float() - ref[k].float()).abs().max() <= 1e-3, k
