"""Seeded token-id streams and the synthetic vocabulary-compression table.

* ``zipf_ids``: ids drawn from a finite Zipf law p(rank r) ~ r^-s over ``vocab`` ids, with
  the rank-to-id assignment given by a seeded permutation (so frequent ids are scattered
  over the vocabulary, as in a real tokenizer).
* ``uniform_ids``: ids uniform over the vocabulary.
* ``phrase_stream``: a Zipf stream in which a target fraction of positions is covered by
  verbatim copies of phrases from a fixed seeded phrase set (heavy n-gram reuse).
* ``remap_table``: a many-to-one, onto map [0, V) -> [0, V'): a seeded permutation pi;
  ids pi[0..V'-1] map one-to-one onto 0..V'-1, every other id maps to a seeded uniform
  target.  It stands in for NFKC + lower-casing equivalence classes, which need a real
  tokenizer vocabulary.
"""
from __future__ import annotations

import numpy as np


def _zipf_cdf(vocab: int, s: float) -> np.ndarray:
    ranks = np.arange(1, vocab + 1, dtype=np.float64)
    w = ranks ** (-float(s))
    cdf = np.cumsum(w)
    return cdf / cdf[-1]


def zipf_ids(vocab: int, s: float, shape, seed: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    perm = rng.permutation(vocab).astype(np.int32)
    cdf = _zipf_cdf(vocab, s)
    n = int(np.prod(shape))
    u = rng.random(n)
    ranks = np.minimum(np.searchsorted(cdf, u, side="right"), vocab - 1)
    return perm[ranks].reshape(shape).astype(np.int32)


def uniform_ids(vocab: int, shape, seed: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(0, vocab, size=shape, dtype=np.int64).astype(np.int32)


def remap_table(vocab_in: int, vocab_out: int, seed: int) -> np.ndarray:
    if not 0 < vocab_out <= vocab_in:
        raise ValueError("need 0 < vocab_out <= vocab_in")
    rng = np.random.Generator(np.random.PCG64(seed))
    perm = rng.permutation(vocab_in)
    table = np.empty(vocab_in, dtype=np.int32)
    table[perm[:vocab_out]] = np.arange(vocab_out, dtype=np.int32)
    rest = perm[vocab_out:]
    table[rest] = rng.integers(0, vocab_out, size=rest.size, dtype=np.int64).astype(np.int32)
    return table


def phrase_stream(vocab: int, s: float, B: int, T: int, seed: int, n_phrases: int = 5000,
                  min_len: int = 4, max_len: int = 16, coverage: float = 0.30) -> np.ndarray:
    """[B, T] ids: Zipf background with ``coverage`` of positions copied from phrases.

    Phrases: ``n_phrases`` fixed sequences, lengths uniform in [min_len, max_len], ids Zipf.
    At each step a phrase is inserted with probability q, else one background token; q is
    chosen so that the expected covered fraction equals ``coverage``.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = rng.integers(min_len, max_len + 1, size=n_phrases)
    total = int(lens.sum())
    pool = zipf_ids(vocab, s, (total,), seed + 7919)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    mean_len = (min_len + max_len) / 2.0
    q = coverage / (mean_len - coverage * (mean_len - 1.0))
    background = zipf_ids(vocab, s, (B * T * 2 + 64,), seed + 104729)
    out = np.empty((B, T), dtype=np.int32)
    bg = 0
    for b in range(B):
        t = 0
        row = out[b]
        while t < T:
            if rng.random() < q:
                p = int(rng.integers(0, n_phrases))
                L = min(int(lens[p]), T - t)
                row[t:t + L] = pool[starts[p]:starts[p] + L]
                t += L
            else:
                row[t] = background[bg]
                bg += 1
                t += 1
    return out
