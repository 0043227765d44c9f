"""Write oracle_tiny_decode.json next to this file: the fp64 oracle's
free-running decode of the `tiny` workload and of its no-cache variant.
The inputs are seeded and synthetic: one layer, d 128, V 1024, 64 prompt
positions and 32 generated in blocks of 8. Each variant is recorded with and
without the bf16 storage rounding.

The fixture is a regression pin of the oracle itself. The pages print no
worked example for the step, so no value here comes from them: every value
is the oracle's, and this script calls nothing but the oracle and the seeded
input generators. tests/test_oracle_golden.py recomputes the decodes and
compares. Regenerate the fixture only together with an intended change to
the oracle's arithmetic, and name in that commit the passage or reading that
justifies the change.

Run from the repository root:  python tests/golden/make_oracle_tiny.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from diffusion_decoding_step_b200 import workload as wl  # noqa: E402
from tests.oracle_inputs import Case  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny_decode.json")
VARIANTS = {"tiny_prefix": wl.WORKLOADS["tiny"],
            "tiny_nocache": wl.WORKLOADS["tiny"].replace(mode=wl.MODE_NONE)}


def record(w, mirror):
    """The decode as plain lists: steps per block, final generated tokens, and
    per step the block start, committed positions, tokens and confidences
    (null where the row was not masked)."""
    tr = Case(w).decode(mirror=mirror)
    steps = []
    for s, r in tr.steps:
        conf = [None if np.isnan(c) else float(c) for c in r.conf[0]]
        steps.append({"block": int(s), "commit": [int(i) for i in np.flatnonzero(r.commit[0])],
                      "tok": [int(t) for t in r.tok[0]], "conf": conf})
    return {"steps_per_block": [int(n) for n in tr.steps_per_block],
            "tokens": [int(t) for t in tr.tokens[0, w.prompt_len:]], "steps": steps}


def main():
    out = {}
    for name, w in VARIANTS.items():
        for mirror in (True, False):
            out[f"{name}:{'mirror' if mirror else 'exact'}"] = record(w, mirror)
    with open(OUT, "w") as f:   # one line per step
        f.write("{\n")
        for i, (key, rec) in enumerate(sorted(out.items())):
            f.write(f' "{key}": {{"steps_per_block": {json.dumps(rec["steps_per_block"])},\n')
            f.write(f'  "tokens": {json.dumps(rec["tokens"])},\n  "steps": [\n')
            f.write(",\n".join("   " + json.dumps(st, sort_keys=True) for st in rec["steps"]))
            f.write("]}" + ("," if i + 1 < len(out) else "") + "\n")
        f.write("}\n")
    print(OUT)


if __name__ == "__main__":
    main()
