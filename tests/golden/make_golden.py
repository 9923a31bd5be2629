"""Writes tests/golden/long_run_schedule.json from the oracle only (no CUDA path).

The pages print no worked numeric example of the window step, so the only stored
expected values are these schedule facts of the 257-frame run (2-frame blocks, a window
of 8 blocks, 50 evaluations per block, entry of block b at floor(b * 50 / 8)).
Run: python tests/golden/make_golden.py
"""
import collections
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle as O  # noqa: E402


def main():
    sch = O.long_run_schedule(129, 8, 50)
    hist = collections.Counter(len(s["live"]) for s in sch)
    data = {
        "n_steps": len(sch),
        "block_count_histogram": {str(k): hist[k] for k in sorted(hist)},
        "entry_steps_first_10": [O.entry_step(b, 50, 8) for b in range(10)],
        "pop_steps_first_3": [s["step"] for s in sch if s["pop_after"]][:3],
        "n_pops": sum(len(s["pop_after"]) for s in sch),
        "tau_first_5": O.timestep_schedule(50)[:5],
    }
    with open(os.path.join(HERE, "long_run_schedule.json"), "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
        f.write("\n")


if __name__ == "__main__":
    main()
