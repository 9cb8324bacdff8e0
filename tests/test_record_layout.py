"""The record layout that include/tkv.h documents for C callers (element order of
a K or V block: quarters of b 32-bit words, pairs 16 bits apart, pair -> head-dim
maps), checked against the oracle's packing.  The header text is the contract a
caller codes against, so it is read here and restated as a formula; every code of
every dim of every class must sit where the header says."""
from pathlib import Path

import numpy as np
import pytest

from oracle import oracle as orc
from tests.helpers import bf16_bits

ROOT = Path(__file__).resolve().parents[1]


def header_position(bits: int, is_v: bool, dim: int):
    """(byte offset inside the block, bit offset inside the 32-bit word) of head dim
    `dim`, following the header's words: quarter q has `bits` words, word w holds
    pairs p = w*(16/bits) + j, first member at bit bits*j, second 16 bits higher;
    pair p of quarter q holds K dims 32(p/4) + 8q + 2(p%4) + {0,1}, V dims
    8p + 2q + {0,1}."""
    ppw = 16 // bits
    for q in range(4):
        for p in range(16):
            base = 8 * p + 2 * q if is_v else 32 * (p // 4) + 8 * q + 2 * (p % 4)
            if dim in (base, base + 1):
                w, j = p // ppw, p % ppw
                bit = bits * j + (16 if dim == base + 1 else 0)
                return 4 * bits * q + 4 * w, bit
    raise AssertionError(dim)


def test_header_states_the_layout_it_is_checked_against():
    text = (ROOT / "include" / "tkv.h").read_text()
    for phrase in ("K block: 32*(p/4) + 8*q + 2*(p%4) + {0, 1}", "V block: 8*p + 2*q + {0, 1}",
                   "second member 16 bits higher"):
        assert phrase in text, phrase


@pytest.mark.parametrize("bits", [8, 4, 2])
def test_code_positions_match_the_header(bits):
    rng = np.random.default_rng(bits)
    # distinct values inside every group, in a different order per group and per
    # K/V, so that a wrong group or a swapped pair member shows up as a wrong code
    k = np.concatenate([rng.permutation(32) * 0.25 + 8 * g for g in range(4)]).astype(np.float32)
    v = np.concatenate([rng.permutation(32) * 0.5 - 3 * g for g in range(4)]).astype(np.float32)
    kb, vb = bf16_bits(k), bf16_bits(v)
    rec = orc.pack_record(bits, kb, vb)
    cb = 128 * bits // 8
    for is_v, xb, off in ((False, kb, 0), (True, vb, cb)):
        x = xb.astype(np.uint32) << 16
        xf = x.view(np.float32)
        for g in range(4):
            _, _, codes = orc.quantize_group(xf[32 * g:32 * g + 32], bits)
            for j in range(32):
                dim = 32 * g + j
                byte, bit = header_position(bits, is_v, dim)
                word = int.from_bytes(bytes(rec[off + byte:off + byte + 4]), "little")
                got = (word >> bit) & ((1 << bits) - 1)
                assert got == codes[j], (bits, is_v, dim, got, codes[j])


def test_bf16_positions_match_the_header():
    k = np.arange(128, dtype=np.float32) + 1.0
    v = -np.arange(128, dtype=np.float32) - 0.5
    kb, vb = bf16_bits(k), bf16_bits(v)
    rec = orc.pack_record(16, kb, vb)
    for is_v, xb, off in ((False, kb, 0), (True, vb, 256)):
        for dim in range(128):
            byte, bit = header_position(16, is_v, dim)
            word = int.from_bytes(bytes(rec[off + byte:off + byte + 4]), "little")
            assert (word >> bit) & 0xFFFF == int(xb[dim]), (is_v, dim)
