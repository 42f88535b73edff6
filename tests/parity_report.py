"""Table of the GPU parity error statistics logged by the tests.

    GDLA_PARITY_LOG=/tmp/parity.jsonl python -m pytest tests -m gpu
    python tests/parity_report.py /tmp/parity.jsonl > table.md

One row per checked tensor, as tests/parity.py logs it: max, mean and RMS
absolute error against the float64 oracle, max|oracle|, the tolerance
1e-2 * max|oracle| + 1e-3, its margin, and where the largest error sits.
"""
from __future__ import annotations

import json
import sys


def report(path: str) -> str:
    recs = [json.loads(line) for line in open(path) if line.strip()]
    out = ["| checked tensor | elements | max abs err | mean abs err | RMS err | max abs oracle "
           "| tol | err / tol | argmax |",
           "|---|---|---|---|---|---|---|---|---|"]
    worst = 0.0
    for r in recs:
        ratio = r["max_abs_err"] / r["tol"] if r["tol"] else float("inf")
        worst = max(worst, ratio)
        out.append("| %s | %d | %.3e | %.3e | %.3e | %.3f | %.3e | %.3f | %s |" % (
            r["what"], r["elements"], r["max_abs_err"], r["mean_abs_err"], r["rms_err"],
            r["max_abs_ref"], r["tol"], ratio, tuple(r["argmax"])))
    out.append("")
    out.append("%d tensors; largest err / tol = %.3f (1.0 would fail)." % (len(recs), worst))
    return "\n".join(out)


if __name__ == "__main__":
    print(report(sys.argv[1]))
