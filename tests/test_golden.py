"""Stored fixtures: the pages' one piece of arithmetic, and an oracle regression record."""
import json
import os

import numpy as np

import oracle
from mla_flash_attention_attn_b200 import workloads as W

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_page_score_matrix_size():
    rec = json.load(open(os.path.join(HERE, "page_arithmetic.json")))
    nbytes = rec["seq_len"] * rec["seq_len"] * rec["bytes_per_score"]
    assert nbytes == rec["score_matrix_mib"] * 2 ** 20


def test_oracle_regression_record():
    rec = json.load(open(os.path.join(HERE, "oracle_tiny.json")))
    w = W.make("v2lite_decode", n_kv=24, n_head=2, n_pad=5)
    out = oracle.attention(w.q[0], w.kcache[0], mask=w.mask[0], scale=w.scale)
    cols = rec["cols_sampled"]
    for r in range(rec["rows"]):
        got = [float(out[r, c]) for c in cols]
        want = [float(v) for v in rec["values"][r]]
        np.testing.assert_allclose(got, want, rtol=1e-14, atol=0)
