"""Writes tests/golden/dirichlet_factors.txt from the closed form (standard library only).

The amplitude kept by block mean pooling of a constant pair rotated at
frequency theta per position (RoPE) is the Dirichlet factor
    D(theta, beta) = |sin(beta*theta/2)| / (beta * |sin(theta/2)|),
the magnitude of (1/beta) * sum_{u<beta} exp(i*u*theta).  This is the
"destructive interference" / amplitude collapse of
"Prism: Spectral-Aware Block-Sparse Attention", §2.
"""
import math
import pathlib


def dirichlet(theta: float, beta: int) -> float:
    return abs(math.sin(beta * theta / 2)) / (beta * abs(math.sin(theta / 2)))


CASES = [
    # (rope base, head_dim, pair m, block beta)
    (1e4, 64, 0, 64),      # theta = 1 (the highest-frequency pair)
    (5e5, 128, 0, 128),    # theta = 1
    (1e4, 64, 31, 64),     # lowest pair of the 64-dim head: theta = 1e4**(-62/64)
    (1e4, 64, 8, 64),
    (5e5, 128, 16, 128),
    (5e5, 128, 40, 128),
]


def render() -> str:
    lines = ["# Prism: Spectral-Aware Block-Sparse Attention, §2 (mean pooling under RoPE, blind spot)",
             "# D = |sin(beta*theta/2)| / (beta*|sin(theta/2)|), theta = base**(-2m/d); written by make_golden.py",
             "# base head_dim m beta theta D"]
    for base, d, m, beta in CASES:
        theta = base ** (-2.0 * m / d)
        lines.append(f"{base:g} {d} {m} {beta} {theta:.17g} {dirichlet(theta, beta):.12f}")
    return "\n".join(lines) + "\n"


def main():
    pathlib.Path(__file__).with_name("dirichlet_factors.txt").write_text(render())


if __name__ == "__main__":
    main()
