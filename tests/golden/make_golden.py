"""Writes tests/golden/fig2_sets.json from the oracle alone.

Setting from the LTE paper's Figure 2 caption ("Alleviating Forgetfulness of
Linear Attention by Hybrid Sparse Attention and Contextualized Learnable Token
Eviction"): attention sink s=2, sliding window w=12.  The caption gives no cap
and no mask, so this fixture picks C=4 and a fixed Bernoulli(0.35) mask.
Run: python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))
from oracle import lte_oracle as O  # noqa: E402

T, S, W, C = 40, 2, 12, 4
mask = O.fed_mask((np.random.default_rng(2510).random(T) < 0.35).astype(np.uint8), S)
sets = [O.attended_set(t, mask, S, W, C) for t in range(T)]
out = {"source": "LTE paper, Figure 2 caption: s=2, w=12 (C and mask chosen here)",
       "sink": S, "window": W, "cap": C, "mask": mask.tolist(), "sets": sets}
with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "fig2_sets.json"), "w") as f:
    json.dump(out, f)
print("wrote", len(sets), "rows")
