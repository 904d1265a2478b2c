"""Seeded random streams for rotation, sign and projection generation.

TEST INFRASTRUCTURE (oracle).  Not imported by the product path.

The upstream guide (section 3, Codex finding 6; section 10, open question 2)
asks for rotations generated deterministically from a seed instead of a
static table, and names the property "same seed -> same matrix".  It never
names the generator.  Reading taken here (shared by both implementations, each
written independently from the published definition):

* SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014; the public-domain reference by S. Vigna): the state
  starts at ``seed``; each draw adds the golden-gamma 0x9E3779B97F4A7C15 to the
  state (mod 2^64) and returns the state passed through the two
  xor-shift-multiply rounds and a final xor-shift.
* uniform in [0, 1): the top 53 bits of a draw times 2^-53.
* sign: -1 if the top bit of a draw is set, else +1.
* standard normal: Box-Muller on consecutive uniform pairs (u1, u2) with
  u1 replaced by 1 - u1 so that it lies in (0, 1]; each pair yields
  sqrt(-2 ln u1) cos(2 pi u2) then sqrt(-2 ln u1) sin(2 pi u2), in that order.
"""

import numpy as np

GOLDEN_GAMMA = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB
MASK64 = (1 << 64) - 1


def splitmix64(seed, n):
    """First ``n`` SplitMix64 outputs for ``seed`` as a uint64 array.

    State after draw i (1-based) is seed + i * gamma (mod 2^64), so the
    sequence is evaluated as a vector of states; each goes through the
    output function unchanged.
    """
    with np.errstate(over="ignore"):
        i = np.arange(1, n + 1, dtype=np.uint64)
        z = np.uint64(seed & MASK64) + i * np.uint64(GOLDEN_GAMMA)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(MIX1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(MIX2)
        z = z ^ (z >> np.uint64(31))
    return z


def uniforms(seed, n):
    """``n`` uniforms in [0, 1): (draw >> 11) * 2^-53."""
    z = splitmix64(seed, n)
    return (z >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def signs(seed, n):
    """``n`` signs (+1.0 / -1.0): -1 where the draw's top bit is set."""
    z = splitmix64(seed, n)
    top = (z >> np.uint64(63)).astype(np.int64)
    return np.where(top == 1, -1.0, 1.0)


def gaussians(seed, n):
    """``n`` standard normals by Box-Muller from the uniform stream.

    Pair k uses uniforms 2k (u1) and 2k+1 (u2); u1 := 1 - u1 lies in (0, 1].
    Output 2k is r cos(2 pi u2), output 2k+1 is r sin(2 pi u2),
    r = sqrt(-2 ln u1).
    """
    n_pairs = (n + 1) // 2
    u = uniforms(seed, 2 * n_pairs)
    u1 = 1.0 - u[0::2]
    u2 = u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    g = np.empty(2 * n_pairs, dtype=np.float64)
    g[0::2] = r * np.cos(2.0 * np.pi * u2)
    g[1::2] = r * np.sin(2.0 * np.pi * u2)
    return g[:n]
