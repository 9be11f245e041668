"""Writes the stored expected values under tests/golden/ from the oracle only.

Run from the repository root:  python tests/golden/make_golden.py
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402


def lvsa_tiny(order: str, name: str):
    # LVSA frame sets of the tiny workload (T=8, C=4, T_per=4, steps 0..3),
    # "LVSA: Training-Free Sparse Attention for Long Video Diffusion", section 2
    path = os.path.join(HERE, name)
    with open(path, "w") as f:
        f.write(f"# LVSA frame sets A(t), T=8 C=4 T_per=4, window growth {order!r}; "
                "columns: s t frames...\n")
        for s in range(4):
            A = oracle.lvsa_frame_sets(8, 4, 4, s, order=order)
            for t in range(8):
                f.write(" ".join(str(int(v)) for v in (s, t, *A[t])) + "\n")


if __name__ == "__main__":
    lvsa_tiny("alternate", "lvsa_tiny_T8_C4_Tper4.txt")
    lvsa_tiny("distance", "lvsa_tiny_T8_C4_Tper4_distance.txt")
