"""Seeded random parameters of the quantizer (oracle side; test infrastructure).

The pages fix the distributions but no generator:
  * the rotation is random and seeded; its efficient form is sign flips
    followed by a Walsh-Hadamard transform ("内存厂商的噩梦来了", section 4,
    the note after the pseudocode that names WHT);
  * the QJL projection S has i.i.d. standard normal entries ("TurboQuant của
    Google: nén KV cache 6 lần", section "Vấn đề của inner product", QJL;
    "I Spent 31 Hours On The Math Behind Turboquant", property 1:
    S.x ~ N(0, ||x||^2 I)).

Reading taken here: the counter-based SplitMix64 generator (Steele, Lea and
Flood, OOPSLA 2014; the public-domain splitmix64.c), output k of seed s being
mix(s + (k+1) * 0x9E3779B97F4A7C15).  Signs: +1 when bit 63 of output i is
clear, else -1.  S: row-major, entry e from the Box-Muller pair of outputs
(2*(e//2), 2*(e//2)+1), each mapped to (out >> 11) * 2^-53, the first one
replaced by 1-u so the log never sees zero; cos for even e, sin for odd e;
float64 arithmetic rounded once to fp32.

The dense rotation's Gaussian matrix G (oracle.rotation.haar_matrix) is the
same stream, kept in float64.
"""

import math

import numpy as np

_MASK = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15


def splitmix64(seed: int, k: int) -> int:
    """Output ``k`` (0-based) of SplitMix64 started at ``seed``."""
    z = (seed + (k + 1) * _GAMMA) & _MASK
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK
    return z ^ (z >> 31)


def signs(seed: int, d: int) -> np.ndarray:
    """Rademacher diagonal D of the randomized Hadamard rotation, as int8 +-1."""
    out = np.empty(d, dtype=np.int8)
    for i in range(d):
        out[i] = -1 if (splitmix64(seed, i) >> 63) & 1 else 1
    return out


def _unit53(v: int) -> float:
    return (v >> 11) * (1.0 / 9007199254740992.0)


def gaussian_matrix_f64(seed: int, d: int) -> np.ndarray:
    """d x d i.i.d. N(0,1) entries, row-major, float64 (Box-Muller, unrounded)."""
    n = d * d
    out = np.empty(n, dtype=np.float64)
    for p in range((n + 1) // 2):
        u1 = 1.0 - _unit53(splitmix64(seed, 2 * p))
        u2 = _unit53(splitmix64(seed, 2 * p + 1))
        r = math.sqrt(-2.0 * math.log(u1))
        ang = 2.0 * math.pi * u2
        out[2 * p] = r * math.cos(ang)
        if 2 * p + 1 < n:
            out[2 * p + 1] = r * math.sin(ang)
    return out.reshape(d, d)


def gaussian_matrix(seed: int, d: int) -> np.ndarray:
    """QJL projection S in R^{d x d}, i.i.d. N(0,1), row-major, fp32."""
    return gaussian_matrix_f64(seed, d).astype(np.float32)
