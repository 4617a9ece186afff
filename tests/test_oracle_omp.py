"""The all-cores CPU baseline (oracle/moe_oracle_omp.c) equals the single-threaded oracle.

The variant only splits the tokens of route, permute and combine over OpenMP threads and
calls the unchanged oracle functions on each chunk, so every output must match the serial
oracle bit for bit, for any thread count (a ragged last chunk included)."""

import os
import subprocess
import sys

import pytest


@pytest.mark.parametrize("threads", ["1", "3", "8"])
def test_omp_variant_matches_the_serial_oracle(threads):
    # a fresh process per thread count: OpenMP reads OMP_NUM_THREADS once
    code = f"""
import numpy as np, oracle
from synthetic import get_workload, make_inputs
w = get_workload("tiny").scaled(301)
d = make_inputs(w)
mask = (np.arange(w.N) % 17 == 5).astype(np.uint8)
i1, p1 = oracle.route_topk(d["logits"], w.k, token_mask=mask)
i2, p2 = oracle.omp_route_topk(d["logits"], w.k, token_mask=mask)
assert np.array_equal(i1, i2) and np.array_equal(p1.view(np.uint32), p2.view(np.uint32))
L = oracle.layout(i1, p1, E_log=w.E_log, R=w.R, C=40)
s1 = oracle.permute(d["hidden"], L["dest_row"], L["rows_max"])
s2 = oracle.omp_permute(d["hidden"], L["dest_row"], L["rows_max"])
assert np.array_equal(s1, s2)
for probs in (p1, None):
    assert np.array_equal(oracle.combine(s1, L["dest_row"], probs), oracle.omp_combine(s1, L["dest_row"], probs))
assert oracle.omp_threads() == {threads}
print("ok")
"""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, OMP_NUM_THREADS=threads, PYTHONPATH=root)
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "ok" in r.stdout, r.stderr[-2000:]
