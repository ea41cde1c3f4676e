"""Philox4x32-10 counter-based generator and the noise it feeds (oracle side).

Test infrastructure only (see ``oracle/__init__``).

Philox4x32-10 is written here from its published definition (Salmon, Moraes,
Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11): four 32-bit
counter words, two 32-bit key words, ten rounds; each round multiplies counter
words 0 and 2 by the two Philox multipliers, takes the high halves XOR the
other counter word XOR a key word, and the key is bumped by the two Weyl
constants between rounds.  Pinned by the published known-answer vectors
(tests/golden/philox4x32_10_kat.txt).

The pages fix only *that* sampling is random (the SMC-SD bonus token, the
STAND Gumbel noise "precomputed and cached", STAND Methodology item 2); this
library regenerates the noise from counters instead of caching it, which gives
the same distribution and stores nothing.  Counter layout used by every stream:

    key     = (seed mod 2^32, seed div 2^32)
    counter = (c0, c1, round mod 2^32, tag + 16 * ((round div 2^32) mod 2^28))

with c1 the row / particle / sequence id of the draw and c0 the vocabulary
position divided by 4 (word = position mod 4) for per-entry noise, or c0 = 0,
word 0 for a per-row scalar.
"""

import numpy as np

_MASK = np.uint64(0xFFFFFFFF)
_M0 = np.uint64(0xD2511F53)
_M1 = np.uint64(0xCD9E8D57)
_W0 = np.uint64(0x9E3779B9)
_W1 = np.uint64(0xBB67AE85)
_S32 = np.uint64(32)

# Stream tags (the fourth counter word's low 4 bits).
STREAM_BONUS = 1        # bonus-token Gumbel noise (per vocabulary entry)
STREAM_ACCEPT = 2       # accept/reject uniform of standard SD verify (per row)
STREAM_RESIDUAL = 3     # residual-resample Gumbel noise (per vocabulary entry)
STREAM_RESAMPLE = 4     # systematic-resampling offset u0 (per sequence)
STREAM_TOPK_DENSE = 5   # dense Gumbel-top-k noise (per vocabulary entry)
STREAM_TOPK_SPARSE = 6  # sparse Gumbel-top-k noise (per stored entry)
STREAM_DRAFT = 8        # draft-token Gumbel noise of the draft step (per vocabulary entry)
STREAM_BONUS_BLOCK = 9  # bonus-token Gumbel noise per block of 128 entries (two-level draw)
STREAM_DRAFT_BLOCK = 10  # draft-token Gumbel noise per block of 128 entries (two-level draw)
STREAM_TOPK_BLOCK = 11  # dense Gumbel-top-k: block-maximum noise per block of 128 entries
STREAM_RESIDUAL_BLOCK = 12  # verify residual draw: noise per block of 128 entries (two-level)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Ten Philox4x32 rounds on (broadcastable) uint32-valued arrays.

    Returns the four output words as uint64 arrays holding 32-bit values.
    """
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint64) & _MASK for c in (c0, c1, c2, c3))
    k0 = np.asarray(k0, dtype=np.uint64) & _MASK
    k1 = np.asarray(k1, dtype=np.uint64) & _MASK
    for rnd in range(10):
        p0 = _M0 * c0          # 32x32 -> 64-bit product, exact in uint64
        p1 = _M1 * c2
        c0, c1, c2, c3 = ((p1 >> _S32) ^ c1 ^ k0, p1 & _MASK,
                          (p0 >> _S32) ^ c3 ^ k1, p0 & _MASK)
        if rnd != 9:
            k0 = (k0 + _W0) & _MASK
            k1 = (k1 + _W1) & _MASK
    return c0, c1, c2, c3


def _key_and_counter_tail(seed, rnd, tag):
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    rnd = int(rnd) & 0xFFFFFFFFFFFFFFFF
    k0, k1 = seed & 0xFFFFFFFF, seed >> 32
    c2 = rnd & 0xFFFFFFFF
    c3 = (int(tag) + 16 * ((rnd >> 32) & 0x0FFFFFFF)) & 0xFFFFFFFF
    return k0, k1, c2, c3


def stream_words(seed, rnd, tag, c1, n):
    """32-bit words for positions 0..n-1 of one (row id ``c1``) stream.

    ``c1`` may be an array of row ids (shape [R]); the result then has shape
    [R, n].  Position v uses counter word c0 = v // 4 and output word v % 4.
    """
    k0, k1, c2, c3 = _key_and_counter_tail(seed, rnd, tag)
    c1 = np.asarray(c1, dtype=np.uint64)
    ncalls = (int(n) + 3) // 4
    c0 = np.arange(ncalls, dtype=np.uint64)
    if c1.ndim == 0:
        out = philox4x32_10(c0, c1, c2, c3, k0, k1)
        words = np.stack(out, axis=-1).reshape(-1)
        return words[:n]
    out = philox4x32_10(c0[None, :], c1[:, None], c2, c3, k0, k1)
    words = np.stack(out, axis=-1).reshape(c1.shape[0], -1)
    return words[:, :n]


def row_scalar_word(seed, rnd, tag, c1):
    """Word 0 of the call with c0 = 0: the per-row scalar draw of a stream."""
    k0, k1, c2, c3 = _key_and_counter_tail(seed, rnd, tag)
    out = philox4x32_10(0, np.asarray(c1, dtype=np.uint64), c2, c3, k0, k1)
    return out[0]


def uniform_from_bits(x):
    """u = (floor(x / 2^9) + 1/2) * 2^-23, in [2^-24, 1 - 2^-24], exact in fp64.

    23 random bits and a half-step offset: u never hits 0 or 1, and both u and
    1 - u are exactly representable in fp32 and fp64.
    """
    x = np.asarray(x, dtype=np.uint64)
    return ((x >> np.uint64(9)).astype(np.float64) + 0.5) * (2.0 ** -23)


def gumbel_from_uniform(u):
    """Standard Gumbel variate g = -log(-log u), evaluated accurately in fp64.

    For u > 1/2 the inner log is formed as log1p(-(1 - u)) (1 - u is exact), so
    g keeps full relative accuracy in the right tail where it is large.
    """
    u = np.asarray(u, dtype=np.float64)
    t = np.where(u > 0.5, -np.log1p(-(1.0 - u)), -np.log(u))
    return -np.log(t)


GUMBEL_MIN = float(gumbel_from_uniform(2.0 ** -24))
GUMBEL_MAX = float(gumbel_from_uniform(1.0 - 2.0 ** -24))
