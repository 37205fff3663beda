"""Pins of the dropout oracle (``oracle/dropout_oracle.c``): its Philox4x64-10 against
numpy's Philox bit generator (a library routine), the byte layout through a pure-Python
brute force driven by numpy's generator, the exact reduction to plain attention at
threshold 0, unbiasedness (the mean over seeds approaches attention without dropout) and
the keep fraction 1 - threshold/256.

The page "Flash Attention" (section "Zentrale technische Innovationen", the fusion
bullet) lists dropout among the operations fused with the softmax.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def numpy_block(counter, key):
    """Philox4x64-10 block for `counter` from numpy, whose raw output starts at the block
    after its counter: start it at counter - 1 (a 256-bit number, little-endian words,
    wrapping modulo 2^256 like numpy's counter)."""
    value = (sum(int(w) << (64 * n) for n, w in enumerate(counter)) - 1) % 2**256
    start = np.array([(value >> (64 * n)) & (2**64 - 1) for n in range(4)], dtype=np.uint64)
    return np.random.Philox(counter=start, key=np.array(key, dtype=np.uint64)).random_raw(4)


@pytest.mark.parametrize("counter,key", [
    ([1, 0, 0, 0], [0, 0]), ([6, 7, 9, 11], [0x123456789ABCDEF0, 0x0FEDCBA987654321]),
    ([2**63, 2**40 + 3, 17, 2**64 - 1], [2**64 - 1, 5]), ([1000, 3, 12, 0], [42, 7])])
def test_philox_matches_numpy(counter, key):
    assert np.array_equal(oracle.philox4x64(counter, key), numpy_block(counter, key))


def test_dropout_bytes_follow_the_stated_layout():
    """Key j of row i of (batch, head) bh: byte j mod 32 (little-endian in the four words)
    of the block for counter (j / 32, i, bh, 0) and key (seed, offset)."""
    seed, offset = 1234, 99
    for bh, i, j in [(0, 1, 0), (3, 17, 31), (3, 17, 32), (7, 200, 1000), (1, 5, 63), (2, 0, 7)]:
        block = numpy_block([j // 32, i, bh, 0], [seed, offset])
        t = j % 32
        expect = (int(block[t // 8]) >> (8 * (t % 8))) & 0xFF
        assert oracle.dropout_byte(seed, offset, bh, i, j) == expect


def test_threshold_zero_is_plain_attention():
    q, k, v = rnd((1, 2, 9, 8), 1), rnd((1, 2, 9, 8), 2), rnd((1, 2, 9, 8), 3)
    for causal in (False, True):
        o1, l1 = oracle.attention_dropout_rows(q, k, v, 0.4, causal, 0, 5, 6)
        o2, l2 = oracle.attention_rows(q, k, v, 0.4, causal)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


@pytest.mark.parametrize("causal,nq,nk", [(False, 40, 40), (True, 40, 40), (False, 25, 40),
                                           (True, 25, 40), (True, 40, 25)])
def test_bruteforce_with_numpy_bytes(causal, nq, nk):
    """Causal masks align at the bottom right (key j admissible for query i iff
    j <= i + nk - nq); a row without admissible keys has O = 0 and LSE = -inf."""
    B, H, d, thr, seed, off = 1, 2, 3, 77, 2024, 3
    q, k, v = rnd((B, H, nq, d), 4), rnd((B, H, nk, d), 5), rnd((B, H, nk, d), 6)
    o, lse = oracle.attention_dropout_rows(q, k, v, 0.5, causal, thr, seed, off)
    o, lse = o.reshape(B, H, nq, d), lse.reshape(B, H, nq)
    for h in range(H):
        for i in range(nq):
            keys = range(max(0, min(nk, i + 1 + nk - nq))) if causal else range(nk)
            if len(keys) == 0:
                assert np.all(o[0, h, i] == 0.0) and np.isneginf(lse[0, h, i])
                continue
            e = [math.exp(0.5 * math.fsum(q[0, h, i, t] * k[0, h, j, t] for t in range(d)))
                 for j in keys]
            z = math.fsum(e)
            assert abs(lse[0, h, i] - math.log(z)) < 1e-12
            blocks = {}
            out = [0.0] * d
            for n, j in enumerate(keys):
                c = j // 32
                if c not in blocks:
                    blocks[c] = numpy_block([c, i, h, 0], [seed, off])
                byte = (int(blocks[c][(j % 32) // 8]) >> (8 * (j % 8))) & 0xFF
                if byte >= thr:
                    for t in range(d):
                        out[t] += e[n] * v[0, h, j, t]
            for t in range(d):
                assert abs(o[0, h, i, t] - out[t] / z / (1 - thr / 256)) < 1e-12


def test_mean_over_seeds_is_attention_without_dropout():
    q, k, v = rnd((1, 1, 6, 4), 7), rnd((1, 1, 50, 4), 8), rnd((1, 1, 50, 4), 9)
    plain, _ = oracle.attention_rows(q, k, v, 0.3, False)
    draws = np.stack([oracle.attention_dropout_rows(q, k, v, 0.3, False, 64, s, 0)[0]
                      for s in range(600)])
    se = draws.std(axis=0) / np.sqrt(len(draws))
    assert np.all(np.abs(draws.mean(axis=0) - plain) <= 5 * se + 1e-12)


def test_keep_fraction():
    thr = 96
    kept = sum(oracle.dropout_byte(11, 0, bh, i, j) >= thr
               for bh in range(2) for i in range(20) for j in range(256))
    n = 2 * 20 * 256
    p = 1 - thr / 256
    assert abs(kept / n - p) <= 5 * math.sqrt(p * (1 - p) / n)
