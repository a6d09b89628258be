"""Writes the golden fixtures in this folder from exact rational arithmetic.

impulse_decay_085.txt: the impulse response y_t = Abar^t of a scalar
time-invariant SSM with Abar = 0.85 and Bbar = C = 1 (llms.blog "State Space
Models and Mamba ...", "Global Convolution": Kbar = (C Bbar, C Abar Bbar, ...);
the decay 0.85 is the value on flashpapers "State-Space Models", "Interactive
Walkthrough").  Calls neither the oracle nor the CUDA library.

Run:  python tests/golden/make_golden.py
"""
import os
from fractions import Fraction

HERE = os.path.dirname(os.path.abspath(__file__))


def main():
    lam = Fraction(85, 100)
    T = 24
    with open(os.path.join(HERE, "impulse_decay_085.txt"), "w") as f:
        f.write("# impulse response of a scalar LTI SSM, Abar = 0.85, Bbar = C = 1, x = e_0\n")
        f.write("# y_t = 0.85^t  (llms.blog 'Global Convolution'; flashpapers 'Interactive Walkthrough')\n")
        f.write("# param decay = 0.85\n")
        f.write("# columns: t y_t\n")
        for t in range(T):
            f.write(f"{t} {float(lam ** t)!r}\n")


if __name__ == "__main__":
    main()
