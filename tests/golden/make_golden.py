"""Writes the oracle regression fixtures in this folder.

Run from the repository root: python tests/golden/make_golden.py
Calls only the oracle and the seeded input generator.
"""

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import kap  # noqa: E402
from synth import make_workload  # noqa: E402


def main():
    w = make_workload(1)
    budget = 0.25
    r = kap.kap_proxy(w.q, w.k_pages, w.page_table, w.seqlens, w.num_kv_heads, w.block_size, budget)
    out = {
        "what": "KAP oracle output on the tiny workload (1024 tokens, 2 q heads, 1 kv head, d 64, "
                "b 64, seed 1) at budget 25%; a regression fixture, not a value from the pages",
        "budget": budget,
        "order": r["order"].tolist(),
        "hrm": r["hrm"].tolist(),
        "count": r["count"].tolist(),
    }
    with open(os.path.join(HERE, "tiny_proxy.json"), "w") as f:
        json.dump(out, f)
        f.write("\n")


if __name__ == "__main__":
    main()
