"""Token-recall study of the dual bound against the coordinate-box (Quest)
bound on the seeded workloads (CPU oracle only; test infrastructure).

    python oracle/quest_recall_study.py [workload ...]

Prints one JSON line per workload: token recall and block density of each
screen at the workload's thresholds, and the box screen's recall when it
keeps as many blocks as the dual screen admitted (section 4.3, "Comparison
with Quest" of the Elastic Threshold Attention pages).
"""
import json
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import workloads  # noqa: E402
from oracle import eta_quest_oracle as qo  # noqa: E402


def main(names):
    for name in names or ["c2_single", "c3_long"]:
        wl = workloads.make(name, 0)
        res = qo.recall_study(wl, n_local_blocks=wl.n_local_blocks)
        print(json.dumps({"workload": name, **{k: (round(v, 4) if isinstance(v, float) else v)
                                                 for k, v in res.items()}}), flush=True)


if __name__ == "__main__":
    main(sys.argv[1:])
