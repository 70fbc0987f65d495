"""Writes the oracle fixtures of this folder:

    python tests/golden/make_fixtures.py

The pages print no worked numerical example, so every stored value here comes
from the float64 oracle (oracle/attn_oracle.py) on the seeded inputs of
attention_online_softmax_fwd_b200/inputs.py; nothing comes from the CUDA path.
The fixtures freeze the oracle's answers for two small cases (rounded to 7
significant digits; the outputs are bf16 on the GPU), so that the GPU tests can
compare against stored values and a change to the oracle's arithmetic shows up
as a changed fixture:

* the tiny causal GQA prefill (B 1, Hq 4, Hkv 2, S 128, D 64), every 16th row
  and the last;
* a paged GQA decode with the BLASST tile skip (3 ragged sequences, Hq 8,
  Hkv 2, D 128, 16-token pages, queries scaled by 3, lambda 0.5, split 1024,
  group decisions: 19 of 66 decisions skipped, none within 0.01 of the threshold): the outputs of query heads 0, 3, 5 and 7, every LSE, the
  decision mask and the decision margins.
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from attention_online_softmax_fwd_b200 import inputs as gen  # noqa: E402
from oracle import attn_oracle as orc  # noqa: E402

PREFILL_ROWS = list(range(0, 128, 16)) + [127]
DECODE_HEADS = [0, 3, 5, 7]
DECODE_LENS = [1, 700, 1300]
DECODE_LAMBDA, DECODE_SPLIT = 0.5, 1024


def _r(x):
    return [float(f"{v:.7g}") if np.isfinite(v) else ("-inf" if v < 0 else "inf") for v in np.asarray(x).ravel()]


def decode_case_inputs():
    c = gen.paged_decode_inputs(len(DECODE_LENS), 8, 2, 128, 16, 0, 0, seed=7001, lens=DECODE_LENS)
    c.q = (c.q.float() * 3.0).to(c.q.dtype)
    return c


def tiny_prefill_fixture():
    cfg = gen.CONFIGS["tiny_gqa_prefill"]
    q, k, v = gen.prefill_inputs(cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["S"], cfg["D"], cfg["seed"])
    scale = gen.attn_scale(cfg["D"])
    o, lse = orc.prefill(q, k, v, True, scale)
    return {"case": "tiny_gqa_prefill", "seed": cfg["seed"], "shape": [cfg["B"], cfg["S"], cfg["Hq"], cfg["D"]],
            "Hkv": cfg["Hkv"], "scale": scale, "rows": PREFILL_ROWS,
            "o": _r(o[0, PREFILL_ROWS]), "lse": _r(lse[0][:, PREFILL_ROWS])}


def blasst_decode_fixture():
    c = decode_case_inputs()
    scale = gen.attn_scale(128)
    o, lse, mask, margin = orc.decode_paged_blasst(c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens, 16, scale,
                                                   DECODE_LAMBDA, DECODE_SPLIT)
    vis = mask != 2
    return {"case": "blasst_paged_decode", "seed": 7001, "lens": DECODE_LENS, "Hq": 8, "Hkv": 2, "D": 128,
            "page_size": 16, "q_times": 3.0, "lambda": DECODE_LAMBDA, "split_tokens": DECODE_SPLIT,
            "scale": scale, "heads": DECODE_HEADS, "o": _r(o[:, DECODE_HEADS]), "lse": _r(lse),
            "mask": mask.ravel().tolist(),
            "mask_shape": list(mask.shape), "margin": _r(np.where(vis, margin, np.inf))}


def build():
    return {"note": "float64 oracle outputs on seeded inputs, written by tests/golden/make_fixtures.py",
            "tiny_gqa_prefill": tiny_prefill_fixture(), "blasst_paged_decode": blasst_decode_fixture()}


if __name__ == "__main__":
    with open(os.path.join(HERE, "oracle_fixtures.json"), "w") as f:
        json.dump(build(), f, separators=(",", ":"))
    print("wrote", os.path.join(HERE, "oracle_fixtures.json"))
