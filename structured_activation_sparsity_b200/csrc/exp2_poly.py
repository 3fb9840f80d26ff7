"""Derives the coefficients of the cubic that approximates 2^f on [-1/2, 1/2] in the attention
kernel's FMA-pipe exponential (csrc/attn.cu, exp2_poly).

Method: 2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2] (Cody-Waite style range
reduction); 2^f is replaced by the cubic that interpolates it at the four Chebyshev nodes
cos((2k+1) pi / 8) / 2, k = 0..3 (Chebyshev interpolation keeps the error close to minimax).
The relative error of the cubic is below 1e-4 on the interval.

Run: python structured_activation_sparsity_b200/csrc/exp2_poly.py
"""
import numpy as np


def coefficients():
    k = np.arange(4)
    nodes = 0.5 * np.cos((2 * k + 1) * np.pi / 8)
    c = np.linalg.solve(np.vander(nodes, 4, increasing=True), 2.0 ** nodes)
    return [float(np.float32(x)) for x in c]


if __name__ == "__main__":
    for i, c in enumerate(coefficients()):
        print(f"c{i} = {c!r}f")
