"""bench.py's byte accounting on CPU: the algorithmic bytes that the roofline
divides by, against a hand total and against a brute-force walk of the
visibility rule (a key counts once per sequence and kv head if any query row
of that sequence may see it)."""

import dataclasses
import itertools
import random

import pytest

import bench
from paged_kv_decode_30_b200 import workloads as W


def _visible_by_rule(wl, L):
    """Keys j < L that some row i sees: causal (fixed first position or
    bottom-right) keeps j <= pos_i, a window W > 0 keeps j >= pos_i - W + 1,
    and with causal off the window is measured from L - 1."""
    seen = set()
    for i in range(wl.q_len):
        if wl.causal_offset >= 0:
            pos, causal = wl.causal_offset + i, True
        elif wl.causal_offset == W.CAUSAL_BOTTOM_RIGHT:
            pos, causal = L - wl.q_len + i, True
        else:
            pos, causal = L - 1, False
        for j in range(L):
            if causal and j > pos:
                continue
            if wl.window > 0 and j < pos - wl.window + 1:
                continue
            seen.add(j)
    return len(seen)


def test_headline_bytes_match_the_hand_total():
    # K+V: 128 seq x 8192 keys x 8 kv heads x 128 x 2 B x 2; Q bf16; O, LSE fp32
    total, kv = bench.algorithmic_bytes(W.HEADLINE, [8192] * 128)
    assert kv == 128 * 8192 * 8 * 128 * 2 * 2 == 4_294_967_296
    assert total == kv + 1_048_576 + 2_097_152 + 16_384 == 4_298_129_408


def test_fp8_bytes_are_one_byte_per_element():
    lens = [100, 4099, 10000, 128]
    total, kv = bench.algorithmic_bytes(W.FP8_VERIFY, lens)
    vis = sum(min(L, 4099) for L in lens)
    assert kv == vis * 8 * 128 * 1 * 2
    rows = W.FP8_VERIFY.batch * 4 * 64
    assert total == kv + rows * (128 * 2 + 128 * 4 + 4)


def test_nvfp4_bytes_are_codes_plus_block_scales():
    # a K (or V) row of 128 elements: 64 bytes of e2m1 codes + 8 e4m3 scales
    total, kv = bench.algorithmic_bytes(W.NVFP4_HEADLINE, [8192] * 128)
    assert kv == 128 * 8192 * 8 * (64 + 8) * 2 == 1_207_959_552
    assert total == kv + 1_048_576 + 2_097_152 + 16_384 == 1_211_121_664


@pytest.mark.parametrize("causal_offset,window,q_len", list(itertools.product(
    [W.CAUSAL_OFF, W.CAUSAL_BOTTOM_RIGHT, 0, 5, 40], [0, 1, 7, 33], [1, 4, 8])))
def test_visible_count_matches_the_rule(causal_offset, window, q_len):
    wl = dataclasses.replace(W.VARLEN, causal_offset=causal_offset, window=window, q_len=q_len)
    rnd = random.Random(causal_offset * 1000 + window * 10 + q_len)
    lens = [0, 1, 2, 3, 8, 9] + [rnd.randint(1, 90) for _ in range(10)]
    assert W.visible_token_count(wl, lens) == sum(_visible_by_rule(wl, L) for L in lens)

