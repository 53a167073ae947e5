"""Philox4x32-10 and the method's random draws (oracle side).

Philox4x32-10 is the counter-based generator of Salmon, Moraes, Dror and Shaw,
"Parallel random numbers: as easy as 1, 2, 3" (SC'11).  The pages do not name
a generator; the sampler's random choices (uniform re-noising of unlocked
positions, the laozijiushiniubi.cn article §一 and §四, and the draw of each
position's next token) need one that both sides can evaluate at any counter,
so each side implements this published generator itself.

Counter layout used by the method (c0, c1, c2, c3), key = (lo32(seed), hi32(seed)):
  c0 = element index (vocab id // 4 for the Gumbel draws, else 0)
  c1 = canvas position
  c2 = block * 256 + step
  c3 = (purpose << 24) | canvas index;  purpose 1 = canvas init,
       2 = Gumbel noise, 3 = re-noise.

Pinned by: the generator's published known-answer vectors (tests/golden/
philox4x32_10_kat.txt) and by agreement with the independent C implementation
in synth/ on random counters.
"""

import numpy as np

_M0 = np.uint64(0xD2511F53)
_M1 = np.uint64(0xCD9E8D57)
_W0 = np.uint64(0x9E3779B9)
_W1 = np.uint64(0xBB67AE85)
_MASK = np.uint64(0xFFFFFFFF)
_S32 = np.uint64(32)

PURPOSE_INIT = 1
PURPOSE_GUMBEL = 2
PURPOSE_RENOISE = 3
PURPOSE_AR_GUMBEL = 5   # the autoregressive mode's Gumbel draw (c1 = 0, c2 = the position)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Ten Philox rounds on (broadcastable) arrays of 32-bit words.

    Each round multiplies words 0 and 2 by the two Philox multipliers, mixes
    the high halves with words 1/3 and the round key, and then the key is
    bumped by the Weyl constants.  Returns the four output words (uint64 arrays
    holding 32-bit values)."""
    c0, c1, c2, c3 = (np.asarray(v, dtype=np.uint64) & _MASK for v in (c0, c1, c2, c3))
    k0 = np.asarray(k0, dtype=np.uint64) & _MASK
    k1 = np.asarray(k1, dtype=np.uint64) & _MASK
    for _ in range(10):
        p0 = _M0 * c0
        p1 = _M1 * c2
        hi0, lo0 = p0 >> _S32, p0 & _MASK
        hi1, lo1 = p1 >> _S32, p1 & _MASK
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
        k0 = (k0 + _W0) & _MASK
        k1 = (k1 + _W1) & _MASK
    return c0, c1, c2, c3


def _key(seed):
    seed = int(seed)
    return seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF


def method_draw(seed, purpose, canvas, block, step, position, c0=0):
    """The four Philox words for one of the method's draws (layout above)."""
    k0, k1 = _key(seed)
    c2 = np.uint64(block * 256 + step)
    c3 = np.uint64((purpose << 24) | canvas)
    return philox4x32_10(c0, position, c2, c3, k0, k1)


def uniform_token(word0, vocab):
    """Uniform token id in [0, V) from one 32-bit word: floor(r * V / 2^32)."""
    return ((np.asarray(word0, dtype=np.uint64) * np.uint64(vocab)) >> _S32).astype(np.int64)


def gumbel_u(words):
    """Uniform variate in (0, 1) from a 32-bit word, exactly representable in
    float32: u = ((r >> 9) + 0.5) * 2^-23."""
    r = np.asarray(words, dtype=np.uint64) >> np.uint64(9)
    return ((r.astype(np.float32) + np.float32(0.5)) * np.float32(2.0 ** -23)).astype(np.float32)


def gumbel_words(seed, canvas, block, step, position, vocab, purpose=PURPOSE_GUMBEL):
    """One 32-bit word per vocabulary id for the Gumbel draw at one position:
    word for id v is output word (v % 4) of the block at c0 = v // 4."""
    n_blocks = (vocab + 3) // 4
    c0 = np.arange(n_blocks, dtype=np.uint64)
    w = method_draw(seed, purpose, canvas, block, step, position, c0)
    return np.stack(w, axis=1).reshape(-1)[:vocab]
