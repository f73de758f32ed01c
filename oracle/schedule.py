"""Calibration-block schedule of the tuning loop (oracle side).

TEST INFRASTRUCTURE ONLY (see the package docstring).

The page "[llm-compressor] AutoRound: 부호 경사 하강법으로 라운딩 최적화"
("on_event with SEQUENTIAL_EPOCH_END") iterates over calibration batches but
does not say how a batch is picked per step.  Reading used here: the n rows form
n / B contiguous blocks of B rows; each epoch visits every block once, in the
order of a Fisher-Yates shuffle (Durstenfeld's in-place form: for i = k-1 down to
1, swap item i with item j = x mod (i + 1)) of the identity permutation, where x
are successive outputs of one SplitMix64 stream seeded with ``seed`` and
continued across epochs.  With a single block no random number is drawn.

SplitMix64 is the generator of Steele, Lea and Flood, "Fast splittable
pseudorandom number generators" (OOPSLA 2014): the state advances by the golden
gamma 0x9E3779B97F4A7C15 and each output is the state passed through the
variant-13 mix (shifts 30, 27, 31; multipliers 0xBF58476D1CE4E5B9 and
0x94D049BB133111EB).
"""
from __future__ import annotations

MASK64 = (1 << 64) - 1
GOLDEN_GAMMA = 0x9E3779B97F4A7C15


def splitmix64_stream(seed: int):
    """Infinite generator of SplitMix64 outputs for the given 64-bit seed."""
    state = seed & MASK64
    while True:
        state = (state + GOLDEN_GAMMA) & MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
        yield z ^ (z >> 31)


def block_schedule(n_blocks: int, iters: int, seed: int) -> list[int]:
    """Block index used at every step t = 0 .. iters-1."""
    if n_blocks < 1:
        raise ValueError("n_blocks must be >= 1")
    if n_blocks == 1:
        return [0] * iters
    rng = splitmix64_stream(seed)
    out: list[int] = []
    while len(out) < iters:
        perm = list(range(n_blocks))
        for i in range(n_blocks - 1, 0, -1):
            j = next(rng) % (i + 1)
            perm[i], perm[j] = perm[j], perm[i]
        out.extend(perm)
    return out[:iters]
