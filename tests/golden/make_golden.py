"""Writes tests/golden/capacities.json from the oracle alone.

Run from the repository root:  python tests/golden/make_golden.py
The capacities follow the reading stated in the oracle: expected rows times the
factor (1.10 sender, 1.15 receiver), rounded up exactly.
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle.moe_oracle import capacities  # noqa: E402

WORKLOADS = {  # T, k, E, D  (three waves each)
    "tiny": (512, 2, 24, 4),
    "mid": (8192, 8, 96, 16),
    "full": (16384, 8, 384, 64),
    "skewed": (65536, 8, 384, 64),
}

if __name__ == "__main__":
    out = {"_about": "Sender / receiver capacities per workload, written by make_golden.py from the oracle.",
           "_factors": "1.10 / 1.15, from 'Marin начинает открытое обучение MoE-модели с 535 млрд параметров', §2"}
    for name, (T, k, E, D) in WORKLOADS.items():
        C_s, C_r = capacities(T, k, E, D, 3)
        out[name] = {"T": T, "k": k, "E": E, "D": D, "W": 3, "C_s": C_s, "C_r": C_r}
    with open(os.path.join(HERE, "capacities.json"), "w", encoding="utf-8") as f:
        json.dump(out, f, indent=1, ensure_ascii=False)
        f.write("\n")
