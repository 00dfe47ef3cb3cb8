"""Write tests/golden/tiny_oracle.json from the oracle alone.

The pages print no worked example, so this fixture holds no page values: it
records the oracle's own outputs on the seeded 64-token workload, so that an
accidental change to the oracle's arithmetic shows up as a test failure.  The
oracle itself is pinned to closed forms, invariants, torch and finite
differences in tests/test_oracle_pins.py.

Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from lm_head_projection_flce_b200 import workloads as W  # noqa: E402  (inputs only)
from oracle import flce_oracle as O  # noqa: E402


def main():
    w = W.TINY
    d = W.generate(w)
    hidden = d["hidden"].double().numpy()
    weight = d["weight"].double().numpy()
    labels = d["labels"].numpy()
    kw = dict(ignore_index=W.IGNORE_INDEX, softcap=w.softcap, unpadded_vocab=w.vocab,
              reduction=w.reduction)
    fwd = O.forward(hidden, weight, labels, **kw)
    dh, dw = O.backward(hidden, weight, labels, **kw)
    out = {
        "workload": w.name,
        "source": "oracle/flce_oracle.py via tests/golden/make_golden.py",
        "loss": fwd.loss,
        "lse_first8": fwd.lse[:8].tolist(),
        "dh_row0_first8": dh[0, :8].tolist(),
        "dw_row_label0_first8": dw[int(labels[labels >= 0][0]), :8].tolist(),
        "dh_abs_sum": float(np.abs(dh).sum()),
        "dw_abs_sum": float(np.abs(dw).sum()),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
