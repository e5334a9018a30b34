"""Write the stored expected thresholds for the large workloads.

Calls only the CPU oracle (``oracle/``) and the seeded input generator
(``workloads/``).  For each workload it stores the oracle's threshold b of
every row it solves, together with digests of the generated inputs so a test
can tell when the generator's output has changed.  The pages print no worked
example, so every stored value here comes from the oracle.

Usage:  python tests/golden/make_golden.py [workload ...]
"""
import json
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from workloads import WORKLOADS, input_digest, make_inputs  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "thresholds.json")
STORED = ["memory_select_256x65536", "adv_mask_3342336", "extreme_1e8"]


def main(names):
    data = {}
    if os.path.exists(OUT):
        with open(OUT) as f:
            data = json.load(f)
    for name in names:
        w = WORKLOADS[name]
        t0 = time.time()
        r, v = make_inputs(w, seed=0)
        b = [oracle.solve_b(row, w.k, w.t) for row in r]
        data[name] = {
            "source": "oracle.solve_b (fp64 full sort + cancellation-free bisection) on "
                      "workloads.make_inputs(seed=0)",
            "B": w.B, "n": w.n, "k": w.k, "t": w.t,
            "digest_r": input_digest(r), "digest_v": input_digest(v),
            "b": b,
        }
        print(f"{name}: {len(b)} rows in {time.time() - t0:.1f} s", flush=True)
        with open(OUT, "w") as f:
            json.dump(data, f, indent=1)
            f.write("\n")


if __name__ == "__main__":
    main(sys.argv[1:] or STORED)
