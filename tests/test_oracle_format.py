"""Pins for the oracle's container and scalar decoders, against things other than
the oracle itself: hand-derived golden blocks, counting arguments, exhaustive
byte round-trips and library fp16/bf16 conversions."""
import itertools
import math
import os

import numpy as np
import pytest

import oracle
from tests.helpers import bf16, f16

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
SYM = {"-": -1, "0": 0, "+": 1}


def _golden(name):
    recs = []
    for line in open(os.path.join(GOLDEN, name)):
        if line.startswith("#") or not line.strip():
            continue
        nm, codes, scale, blk = [p.strip() for p in line.split("|")]
        recs.append((nm, np.array([SYM[c] for c in codes], np.int8), int(scale, 16), bytes.fromhex(blk)))
    return recs


@pytest.mark.parametrize("fmt,fname", [(oracle.PQ2_0, "pq2_blocks.txt"), (oracle.PTQ1_0, "ptq1_blocks.txt")])
def test_golden_blocks(fmt, fname):
    recs = _golden(fname)
    assert len(recs) == 6
    for nm, codes, scale, blk in recs:
        got = oracle.pack(fmt, codes[None, :], np.array([scale], np.uint16))
        assert got.tobytes() == blk, nm
        c2, s2, st = oracle.unpack(fmt, np.frombuffer(blk, np.uint8)[None, :])
        assert st == 0
        np.testing.assert_array_equal(c2[0], codes, err_msg=nm)
        assert int(s2[0, 0]) == scale


def test_block_sizes_and_entropy_floor():
    # "Scion-35B-A3B" card, Weight Representation: 2.125 bpw; FlashNext card: 28 B / 128 = 1.75 bpw.
    assert oracle.block_bytes(oracle.PQ2_0) == 34 and 34 * 8 / 128 == 2.125
    assert oracle.block_bytes(oracle.PTQ1_0) == 28 and 28 * 8 / 128 == 1.75
    # Code bits per group: PQ2 256 >= PTQ1 208 >= 128 log2 3 (the ternary entropy, 1.585 bpw).
    floor = 128 * math.log2(3)
    assert 32 * 8 >= 26 * 8 >= floor
    assert abs(math.log2(3) - 1.585) < 1e-3
    # FlashNext card, Highlights: container overhead about 10% over the entropy.
    assert abs(1.75 / math.log2(3) - 1.104) < 1e-3
    # 3^5 = 243 <= 256 (five trits per byte) and 3^3 = 27 (three trits in the tail byte).
    assert 3 ** 5 <= 256 < 3 ** 6 and 25 * 5 + 3 == 128


def test_pq2_every_byte():
    """All 256 values of one code byte: 3^4 = 81 decode cleanly, the other 175 hold a 3."""
    valid = []
    for b in range(256):
        blk = np.full((1, 34), 0x55, np.uint8)
        blk[0, 0] = b
        codes, _, st = oracle.unpack(oracle.PQ2_0, blk)
        if st == 0:
            valid.append(tuple(codes[0, :4]))
            again = oracle.pack(oracle.PQ2_0, codes, np.zeros((1, 1), np.uint16))
            assert again[0, 0] == b
        else:
            assert st == oracle.EFORMAT
    assert len(valid) == 81
    assert set(valid) == set(itertools.product((-1, 0, 1), repeat=4))


def test_ptq1_every_byte():
    """Quintet byte: 243 valid values, a bijection onto {-1,0,1}^5; tail byte: 27 valid."""
    valid = []
    for b in range(256):
        blk = np.full((1, 28), 0x79, np.uint8)
        blk[0, 25] = 0x0D
        blk[0, 3] = b
        codes, _, st = oracle.unpack(oracle.PTQ1_0, blk)
        if st == 0:
            valid.append(tuple(codes[0, 15:20]))
            again = oracle.pack(oracle.PTQ1_0, codes, np.zeros((1, 1), np.uint16))
            assert again[0, 3] == b
        else:
            assert st == oracle.EFORMAT and b > 242
    assert len(valid) == 243
    assert set(valid) == set(itertools.product((-1, 0, 1), repeat=5))
    tails = []
    for b in range(256):
        blk = np.full((1, 28), 0x79, np.uint8)
        blk[0, 25] = b
        codes, _, st = oracle.unpack(oracle.PTQ1_0, blk)
        if st == 0:
            tails.append(tuple(codes[0, 125:]))
        else:
            assert b > 26
    assert len(tails) == 27 and set(tails) == set(itertools.product((-1, 0, 1), repeat=3))


@pytest.mark.parametrize("fmt", [oracle.PQ2_0, oracle.PTQ1_0])
def test_random_round_trip(fmt):
    rng = np.random.default_rng(5)
    codes = rng.integers(-1, 2, size=(37, 1024)).astype(np.int8)
    scales = rng.integers(0, 1 << 16, size=(37, 8)).astype(np.uint16)
    blocks = oracle.pack(fmt, codes, scales)
    assert blocks.shape == (37, 8 * oracle.block_bytes(fmt))
    c2, s2, st = oracle.unpack(fmt, blocks)
    assert st == 0
    np.testing.assert_array_equal(c2, codes)
    np.testing.assert_array_equal(s2, scales)
    # A random valid byte stream survives unpack -> pack unchanged.
    again = oracle.pack(fmt, c2, s2)
    np.testing.assert_array_equal(again, blocks)


def test_pack_rejects_out_of_range_codes():
    codes = np.zeros((1, 128), np.int8)
    codes[0, 5] = 2
    with pytest.raises(ValueError):
        oracle.pack(oracle.PQ2_0, codes, np.zeros((1, 1), np.uint16))
    with pytest.raises(ValueError):
        oracle.pack(oracle.PTQ1_0, codes, np.zeros((1, 1), np.uint16))


def test_f16_decoder_exhaustive():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = f16(bits)
    got = np.array([oracle.f16_to_f64(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    # Hand values: 0x3C00 = 1, 0x2000 = 2^-7, 0x211F = 1311 * 2^-17, 0x0001 = 2^-24, 0xBC00 = -1.
    assert oracle.f16_to_f64(0x3C00) == 1.0
    assert oracle.f16_to_f64(0x2000) == 2.0 ** -7
    assert oracle.f16_to_f64(0x211F) == 1311 * 2.0 ** -17
    assert oracle.f16_to_f64(0x0001) == 2.0 ** -24
    assert oracle.f16_to_f64(0xBC00) == -1.0


def test_bf16_decoder_exhaustive():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bf16(bits)
    got = np.array([oracle.bf16_to_f64(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    assert oracle.bf16_to_f64(0x3F80) == 1.0 and oracle.bf16_to_f64(0xC000) == -2.0


@pytest.mark.parametrize("fmt", [oracle.PQ2_0, oracle.PTQ1_0])
def test_dequant_row_is_code_times_scale(fmt):
    rng = np.random.default_rng(11)
    codes = rng.integers(-1, 2, size=(3, 384)).astype(np.int8)
    scales = rng.uniform(0.005, 0.02, size=(3, 3)).astype(np.float16).view(np.uint16)
    w = oracle.dequant_rows(fmt, oracle.pack(fmt, codes, scales), 384)
    ref = codes.astype(np.float64) * np.repeat(f16(scales), 128, axis=1)
    np.testing.assert_array_equal(w, ref)
