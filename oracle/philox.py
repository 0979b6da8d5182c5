"""Philox4x32-10 counter-based generator, written from its published definition.

TEST INFRASTRUCTURE ONLY: this module belongs to the CPU oracle.  Only the test
suite, the smoke check and the benchmark's CPU-baseline leg may import it.

Definition followed: J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw,
"Parallel Random Numbers: As Easy as 1, 2, 3", SC'11, section 3.3 (the Philox
S-box: two 32x32->64 multiplies per round, the high halves XORed with the
other two counter words and the round key, the key bumped by the golden-ratio
and sqrt(3)-1 Weyl constants between rounds).  Ten rounds.

Two forms: a scalar one on Python integers (slow, obviously correct, used for
the known-answer pins) and a NumPy one that evaluates many counters at once on
uint64 arrays holding 32-bit values (used by the sampler oracle).  A test pins
the second to the first.

How the denoising sampler keys its draws (a reading; the sampling pages name
only "Philox keyed by seed, block, step and position"):
    key     = (seed, b)                        b = sequence index in the batch
    counter = (j, pos | tag << 24, step, block)
    draw    = output word w of that block
For a per-vocabulary draw at vocabulary index v: j = v >> 2 and w = v & 3.
For a per-position draw (re-noise token, canvas initialisation): j = 0, w = 0.
"""
import numpy as np

MASK32 = 0xFFFFFFFF
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
ROUNDS = 10

TAG_GUMBEL = 0
TAG_RENOISE = 1
TAG_INIT = 2


def philox4x32_10(ctr, key):
    """Scalar Philox4x32-10.  ctr: 4 ints, key: 2 ints (each < 2**32)."""
    c0, c1, c2, c3 = (int(x) & MASK32 for x in ctr)
    k0, k1 = (int(x) & MASK32 for x in key)
    for _ in range(ROUNDS):
        p0 = PHILOX_M0 * c0
        p1 = PHILOX_M1 * c2
        hi0, lo0 = p0 >> 32, p0 & MASK32
        hi1, lo1 = p1 >> 32, p1 & MASK32
        c0, c1, c2, c3 = (hi1 ^ c1 ^ k0) & MASK32, lo1, (hi0 ^ c3 ^ k1) & MASK32, lo0
        k0 = (k0 + PHILOX_W0) & MASK32
        k1 = (k1 + PHILOX_W1) & MASK32
    return (c0, c1, c2, c3)


def philox4x32_10_np(c0, c1, c2, c3, k0, k1):
    """Vectorised Philox4x32-10 over broadcastable arrays of 32-bit values.

    Returns four uint64 arrays holding the 32-bit output words.
    """
    m32 = np.uint64(MASK32)
    c0 = np.asarray(c0, dtype=np.uint64) & m32
    c1 = np.asarray(c1, dtype=np.uint64) & m32
    c2 = np.asarray(c2, dtype=np.uint64) & m32
    c3 = np.asarray(c3, dtype=np.uint64) & m32
    k0 = int(k0) & MASK32
    k1 = int(k1) & MASK32
    c0, c1, c2, c3 = np.broadcast_arrays(c0, c1, c2, c3)
    c0, c1, c2, c3 = (x.copy() for x in (c0, c1, c2, c3))
    M0 = np.uint64(PHILOX_M0)
    M1 = np.uint64(PHILOX_M1)
    s32 = np.uint64(32)
    for _ in range(ROUNDS):
        p0 = M0 * c0  # < 2**64, exact in uint64
        p1 = M1 * c2
        hi0, lo0 = p0 >> s32, p0 & m32
        hi1, lo1 = p1 >> s32, p1 & m32
        c0, c1, c2, c3 = hi1 ^ c1 ^ np.uint64(k0), lo1, hi0 ^ c3 ^ np.uint64(k1), lo0
        k0 = (k0 + PHILOX_W0) & MASK32
        k1 = (k1 + PHILOX_W1) & MASK32
    return c0, c1, c2, c3


def counter_word1(pos, tag):
    """Second counter word: position in the low 24 bits, draw tag above."""
    return (int(pos) & 0xFFFFFF) | (int(tag) << 24)


def uniform_from_word(r):
    """Map a 32-bit word to an open-interval uniform, exactly representable in fp32.

    u = (2 * (r >> 9) + 1) * 2**-24, i.e. the odd multiples of 2**-24 in (0, 1).
    Both u and 1 - u are exact in single precision, so the sampler's transform
    -ln(u) can be evaluated accurately on either side of 1/2.
    """
    r = np.asarray(r, dtype=np.uint64)
    k = (r >> np.uint64(9)).astype(np.float64)
    return (2.0 * k + 1.0) * (2.0 ** -24)


def token_from_word(r, vocab):
    """Uniform token id in [0, vocab): the high half of the 64-bit product r * vocab."""
    r = np.asarray(r, dtype=np.uint64)
    return ((r * np.uint64(vocab)) >> np.uint64(32)).astype(np.int64)


def vocab_words(seed, b, block, step, pos, tag, vocab):
    """Philox words for every vocabulary index v of one (sequence, position) draw row."""
    n_blocks = (vocab + 3) // 4
    j = np.arange(n_blocks, dtype=np.uint64)
    w = philox4x32_10_np(j, counter_word1(pos, tag), step, block, seed, b)
    out = np.stack(w, axis=1).reshape(-1)[:vocab]
    return out


def position_word(seed, b, block, step, pos, tag):
    """The single Philox word used for a per-position draw."""
    return philox4x32_10((0, counter_word1(pos, tag), step, block), (seed, b))[0]
