"""Writes closed_forms.json: tiny attention problems whose result has a closed form.

Expected values come from the formulas below (Python ``math`` only), never from
the oracle or the CUDA library.  sigma(x) = 1 / (1 + exp(-x)).

  two_key_sigmoid   scores (1, 0): p = (sigma(1), 1 - sigma(1)); O = 2 p0 - p1; L = ln(1 + e)
  causal_two_rows   row 0 sees key 0 only: O = v0, L = s00 = 1; row 1 as above
  equal_scores      three equal scores 1: O = mean(v) = 7/3, L = 1 + ln 3
  gqa_two_heads     one K/V head shared by two query heads, scale 1/2:
                    head 0 scores (1, 0), head 1 scores (0, 1)
Run:  python tests/golden/make_closed_forms.py
"""
import json
import math
import os

s1 = 1.0 / (1.0 + math.exp(-1.0))
ln1e = math.log(1.0 + math.e)

cases = [
    {"name": "two_key_sigmoid", "scale": 1.0, "causal": False,
     "q": [[[[1.0]]]], "k": [[[[1.0]], [[0.0]]]], "v": [[[[2.0]], [[-1.0]]]],
     "o": [[[[2.0 * s1 - (1.0 - s1)]]]], "lse": [[[ln1e]]]},
    {"name": "causal_two_rows", "scale": 1.0, "causal": True,
     "q": [[[[1.0]], [[1.0]]]], "k": [[[[1.0]], [[0.0]]]], "v": [[[[2.0]], [[-1.0]]]],
     "o": [[[[2.0]], [[2.0 * s1 - (1.0 - s1)]]]], "lse": [[[1.0, ln1e]]]},
    {"name": "equal_scores", "scale": 1.0, "causal": False,
     "q": [[[[0.5]]]], "k": [[[[2.0]], [[2.0]], [[2.0]]]], "v": [[[[1.0]], [[2.0]], [[4.0]]]],
     "o": [[[[7.0 / 3.0]]]], "lse": [[[1.0 + math.log(3.0)]]]},
    {"name": "gqa_two_heads", "scale": 0.5, "causal": False,
     "q": [[[[1.0, 0.0], [0.0, 1.0]]]], "k": [[[[2.0, 0.0]], [[0.0, 2.0]]]],
     "v": [[[[1.0, 0.0]], [[0.0, 1.0]]]],
     "o": [[[[s1, 1.0 - s1], [1.0 - s1, s1]]]], "lse": [[[ln1e], [ln1e]]]},
]

doc = {"about": "closed-form attention cases; shapes q [B,Lq,Hq,D], k/v [B,Lk,Hkv,D], "
                "o [B,Lq,Hq,D], lse [B,Hq,Lq] (natural log); written by make_closed_forms.py",
       "cases": cases}
with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "closed_forms.json"), "w") as f:
    json.dump(doc, f, indent=1)
