"""Counter-based random stream for the random matrices Pi and S (oracle side).

[TQN] "生成随机旋转矩阵" draws the rotation from ``np.random.randn(d, d)``; the pages
fix no generator.  Reading: a generator defined by publication so that the CUDA
library's host code and this oracle can each implement it independently and draw
the same matrices from the same seed:

* SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number generators",
  OOPSLA 2014): output i (i = 0, 1, ...) is mix(seed + (i + 1) * 0x9E3779B97F4A7C15)
  modulo 2^64, with mix(z) = z ^ (z >> 31) after z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
  and z = (z ^ (z >> 27)) * 0x94D049BB133111EB.
* uniform in (0, 1]:  ((w >> 11) + 1) * 2^-53.
* Box-Muller: Gaussian pair j uses uniforms (u_{2j}, u_{2j+1}):
  g_{2j} = sqrt(-2 ln u_{2j}) cos(2 pi u_{2j+1}),  g_{2j+1} = sqrt(-2 ln u_{2j}) sin(2 pi u_{2j+1}).
"""
from __future__ import annotations

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
MUL1 = np.uint64(0xBF58476D1CE4E5B9)
MUL2 = np.uint64(0x94D049BB133111EB)


def splitmix64(seed: int, count: int, start: int = 0) -> np.ndarray:
    """Outputs ``start .. start+count-1`` of the SplitMix64 sequence seeded with ``seed``."""
    i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + i * GAMMA
        z = (z ^ (z >> np.uint64(30))) * MUL1
        z = (z ^ (z >> np.uint64(27))) * MUL2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform01(words: np.ndarray) -> np.ndarray:
    """Map 64-bit words to doubles in (0, 1]."""
    return ((words >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)


def gaussian_stream(seed: int, count: int) -> np.ndarray:
    """First ``count`` standard normal draws of the stream (Box-Muller on SplitMix64)."""
    pairs = (count + 1) // 2
    u = uniform01(splitmix64(seed, 2 * pairs))
    u1 = u[0::2]
    u2 = u[1::2]
    rad = np.sqrt(-2.0 * np.log(u1))
    ang = 2.0 * np.pi * u2
    g = np.empty(2 * pairs, dtype=np.float64)
    g[0::2] = rad * np.cos(ang)
    g[1::2] = rad * np.sin(ang)
    return g[:count]
