"""Writes the stored expected values under tests/golden/ from the oracle only.

    python tests/golden/make_golden.py

* oracle_small.json: a few output rows of a seeded small problem (jagged, with
  position and time bias), so that an unintended change of the oracle shows.
* time_bucket_thresholds.txt: for k = 1..127 the smallest |dt| whose bucket
  min(127, floor(ln(max(1,|dt|))/0.301)) is >= k, found by binary search on
  the oracle's own bucket function.  The CUDA library builds its threshold
  table independently; a test compares the two.
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import hstu_inputs as hi  # noqa: E402
import oracle  # noqa: E402


def thresholds(nb=128):
    out = []
    for kk in range(1, nb):
        lo, hi_ = 1, 2 ** 63 - 1
        while lo < hi_:
            mid = (lo + hi_) // 2
            if oracle.time_bucket(mid, nb) >= kk:
                hi_ = mid
            else:
                lo = mid + 1
        out.append(lo)
    return out


def main():
    spec = dict(name="golden", dtype="f32", batch=3, heads=2, d_qk=8, d_v=8,
                lengths=[5, 11, 2], qk_std=0.8, vu_std=1.0, rab_pos_len=11,
                rab_time=True, rab_std=0.3, norm="own")
    inp = hi.make_inputs(hi.Spec(**spec), seed=7)
    y = oracle.fwd(inp)["y"]
    rows = [0, 4, 5, 10, 15, 16, 17]
    buckets = [[dt, oracle.time_bucket(dt)] for dt in
               (0, 1, 2, 3, 7, 20, 299, 300, 301, 86400, 10 ** 6, 10 ** 9, 10 ** 17)]
    with open(os.path.join(HERE, "oracle_small.json"), "w") as f:
        json.dump(dict(source="written by tests/golden/make_golden.py from the fp64 oracle",
                       spec=spec, seed=7, rows=rows, y_rows=y[rows].tolist(),
                       buckets=buckets), f, indent=1)
    with open(os.path.join(HERE, "time_bucket_thresholds.txt"), "w") as f:
        f.write("# k  smallest |dt| with bucket >= k  (written by make_golden.py from the oracle)\n")
        for kk, t in enumerate(thresholds(), start=1):
            f.write("%d %d\n" % (kk, t))


if __name__ == "__main__":
    main()
