"""Write tests/golden/oracle_samples.json: sampled oracle outputs on seeded workloads.

Calls only the oracle and the seeded input generators.  Re-run it only when
the input recipe changes; a change in the stored values otherwise means the
oracle's arithmetic changed.
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from gtr_inputs import WORKLOADS, make_inputs  # noqa: E402

CASES = [
    dict(workload="tiny", direction=0, override={}),
    dict(workload="640", direction=1, override={}),
    dict(workload="640", direction=2, override={"heads": 2}),
    dict(workload="stack", direction=3, override={"B": 1, "heads": 1}),
]


def main():
    fixtures = []
    for i, case in enumerate(CASES):
        w = WORKLOADS[case["workload"]].with_(**case["override"])
        seed = w.seed(case["direction"])
        q, k, v, lg = make_inputs(w, seed)
        out = oracle.gla_fwd(q, k, v, lg, w.H, w.W, case["direction"])
        rng = np.random.default_rng(1234 + i)
        idx = np.stack([rng.integers(0, n, 32) for n in out.shape], axis=1)
        fixtures.append(dict(
            workload=case["workload"], override=case["override"], seed=seed,
            direction=case["direction"], index=idx.tolist(),
            value=[float(out[tuple(r)]) for r in idx],
            rms=float(np.sqrt(np.mean(out ** 2))),
        ))
    with open(os.path.join(HERE, "oracle_samples.json"), "w") as f:
        json.dump(fixtures, f, indent=1)


if __name__ == "__main__":
    main()
