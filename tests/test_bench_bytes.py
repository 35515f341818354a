"""The roofline numerators of the bench: algorithmic bytes of one decode step
written out term by term for the workload shapes (indexer keys of every
cached token, the M gathered K and V rows, the fp32 state read and written,
and the step's own small tensors), independently of the bench's helper."""

import numpy as np

import bench
from lisa_inputs import get_config


def _by_hand(B, Hq, Hkv, d, HI, dI, M, L):
    keys = Hkv * L * dI * 2                        # bf16 indexer key of every cached token
    gather = Hkv * min(M, L) * 2 * d * 2           # selected K and V rows
    state = Hq * d * d * 4 * 2                     # fp32 state read + write
    small = (Hq * d * 2 + 4 * Hkv * d * 2 + 2 * Hkv * dI * 2 + HI * dI * 2 + HI * 4 + Hq * 4 + Hq * d * 2)
    return B * (keys + gather + state + small)


def test_decode_1p5b_16k_bytes():
    cfg = get_config("decode_1p5b_16k")
    got = bench.algorithmic_bytes(cfg, cfg.L)
    assert got == _by_hand(1, 12, 2, 128, 4, 64, 256, 16384)
    assert got == 4194304 + 262144 + 1572864 + 9280 == 6038592


def test_ragged_and_long_decode_bytes():
    cfg = get_config("ragged_7b_b32")
    lengths = np.array([4096, 16384, 200, 9001])
    got = bench._decode_bytes(cfg, lengths, B=len(lengths))
    want = sum(_by_hand(1, 28, 4, 128, 4, 64, 256, int(L)) for L in lengths)
    assert got == want
    cfg5 = get_config("longcot_7b_28l")
    assert bench._decode_bytes(cfg5, 16385) == _by_hand(8, 28, 4, 128, 4, 64, 256, 16385)


def test_short_prefix_gathers_only_its_rows():
    cfg = get_config("decode_1p5b_16k")
    assert bench.algorithmic_bytes(cfg, 100) == _by_hand(1, 12, 2, 128, 4, 64, 256, 100)
