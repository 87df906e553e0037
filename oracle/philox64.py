"""Counter-based Gaussian draws for the initial Q, float64 CPU side.

TEST INFRASTRUCTURE ONLY (see the header of oracle/powersgd64.py).

The initial warm start Q0 ~ N(0, 1) is the one random draw of the method.
Tests normally pass Q0 in as an input; this module exists so that the
library's own seeded draw can be checked element by element.  It restates
two published definitions:

  * Philox4x64-10: Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
    easy as 1, 2, 3", SC'11, section 3 (Philox S-box: two 64x64->128
    multiplies per round, the high halves xored with the key and the other
    two counter words; Weyl key schedule; 10 rounds).
  * Box-Muller: Box and Muller, "A note on the generation of random normal
    deviates", Ann. Math. Stat. 29 (1958).

Mapping (a convention of this repository, stated in the C header too):
key = (seed, layer), counter = (b, s, 0, 0) for block b = e // 4 and draw
index s (0 for the initial Q; step number s >= 1 for the fresh Q of a step
without warm start), where e =
j*r + k indexes Q0 (n x r, row-major); word t = e % 4 of the block feeds
normal t.  Each 64-bit word x becomes u = ((x >> 11) + 0.5) * 2^-53 in (0, 1);
words (0, 1) and (2, 3) are Box-Muller pairs: z_even = rho*cos(2*pi*u_odd),
z_odd = rho*sin(2*pi*u_odd), rho = sqrt(-2 ln u_even).  The float64 z is
rounded to float32.
"""
from __future__ import annotations

import math

import numpy as np

MASK64 = (1 << 64) - 1
# Philox4x64 round multipliers and Weyl key increments (SC'11, Table 2 and
# section 3.3: the golden ratio and sqrt(3)-1 in 64-bit fixed point).
PHILOX_M0 = 0xD2E7470EE14C6C93
PHILOX_M1 = 0xCA5A826395121157
PHILOX_W0 = 0x9E3779B97F4A7C15
PHILOX_W1 = 0xBB67AE8584CAA73B


def _mulhilo(a: int, b: int):
    p = a * b
    return p >> 64, p & MASK64


def philox4x64_10(counter, key):
    """Philox4x64 with 10 rounds on a 4-word counter and 2-word key
    (Python ints).  Returns the 4 output words."""
    x0, x1, x2, x3 = (int(c) & MASK64 for c in counter)
    k0, k1 = (int(k) & MASK64 for k in key)
    for rnd in range(10):
        if rnd:
            k0 = (k0 + PHILOX_W0) & MASK64
            k1 = (k1 + PHILOX_W1) & MASK64
        hi0, lo0 = _mulhilo(PHILOX_M0, x0)
        hi1, lo1 = _mulhilo(PHILOX_M1, x2)
        x0, x1, x2, x3 = hi1 ^ x1 ^ k0, lo1, hi0 ^ x3 ^ k1, lo0
    return x0, x1, x2, x3


def _unit(x: int) -> float:
    return ((x >> 11) + 0.5) * (1.0 / 9007199254740992.0)


def box_muller_block(words):
    """Four 64-bit words -> four float64 standard normals."""
    out = []
    for a, b in ((words[0], words[1]), (words[2], words[3])):
        u0, u1 = _unit(a), _unit(b)
        rho = math.sqrt(-2.0 * math.log(u0))
        out.append(rho * math.cos(2.0 * math.pi * u1))
        out.append(rho * math.sin(2.0 * math.pi * u1))
    return out


def initial_q(seed: int, layer: int, n: int, r: int, draw: int = 0) -> np.ndarray:
    """Q for one layer (n x r float32) under the mapping above; draw 0 is
    the initial Q, draw s >= 1 the fresh Q of step s without warm start."""
    total = n * r
    vals = np.empty(total, dtype=np.float64)
    for b in range((total + 3) // 4):
        z = box_muller_block(philox4x64_10((b, draw, 0, 0), (seed, layer)))
        for t in range(4):
            e = 4 * b + t
            if e < total:
                vals[e] = z[t]
    return vals.astype(np.float32).reshape(n, r)
