"""The CUDA path against the stored oracle answers of tests/golden/oracle_fixtures.json
(float64 oracle on seeded inputs, written by tests/golden/make_fixtures.py): the tiny
causal GQA prefill and a paged GQA decode with the BLASST tile skip, compared with
the same tolerances as the live parity tests."""

import json
import os

import numpy as np
import pytest
import torch

import attention_online_softmax_fwd_b200 as ab
from attention_online_softmax_fwd_b200 import inputs as gen
from parity_util import compare_output, compare_skip

pytestmark = pytest.mark.gpu

HERE = os.path.join(os.path.dirname(__file__), "golden")
FIX = json.load(open(os.path.join(HERE, "oracle_fixtures.json")))


def _arr(vals, shape):
    return np.array([float(x) for x in vals]).reshape(shape)


def test_tiny_prefill_against_stored_oracle(cuda_device):
    f = FIX["tiny_gqa_prefill"]
    B, S, Hq, D = f["shape"]
    q, k, v = gen.prefill_inputs(B, Hq, f["Hkv"], S, D, f["seed"])
    o, lse = ab.prefill(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), causal=True, scale=f["scale"])
    torch.cuda.synchronize()
    rows = f["rows"]
    o_ref = _arr(f["o"], (len(rows), Hq, D))
    lse_ref = _arr(f["lse"], (Hq, len(rows)))
    compare_output(o[0, rows], o_ref, lse[0][:, rows], lse_ref, label="tiny prefill vs stored oracle")


def test_blasst_decode_against_stored_oracle(cuda_device):
    import sys
    sys.path.insert(0, HERE)
    from make_fixtures import decode_case_inputs
    f = FIX["blasst_paged_decode"]
    c = decode_case_inputs()
    args = [t.to(cuda_device) for t in (c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens)]
    o, lse, mask = ab.decode_paged_blasst(*args, f["lambda"], scale=f["scale"], split_tokens=f["split_tokens"])
    torch.cuda.synchronize()
    m_ref = np.array(f["mask"], dtype=np.uint8).reshape(f["mask_shape"])
    margin = _arr(f["margin"], f["mask_shape"])
    st = compare_skip(mask, m_ref, margin, label="blasst decode vs stored oracle")
    assert st["tie_mismatches"] == 0, "a tie-band flip: compare against the live oracle instead"
    assert st["skipped"] > 0
    heads = f["heads"]
    n = len(f["lens"])
    o_ref = _arr(f["o"], (n, len(heads), f["D"]))
    lse_ref = _arr(f["lse"], (n, f["Hq"]))
    compare_output(o[:, heads], o_ref, lse, lse_ref, label="blasst decode vs stored oracle")
