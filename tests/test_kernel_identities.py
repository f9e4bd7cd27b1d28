"""The arithmetic identities two kernels rest on, checked in plain Python.

These emulate, bit for bit or index for index, what the kernels do, from the
definitions of the hardware operations involved (a byte permute, and the
operand layout of an m16n8k16 matrix multiply-accumulate); they share no code
with the CUDA path.  GPU parity of the kernels themselves is in the `gpu`
tests.
"""
import struct

import numpy as np
import pytest


# ---------------------------------------------------------------------------
# Q4_0 nibble decode (gathered FFN, Q4_0 weights)
# ---------------------------------------------------------------------------
def byte_perm(x, y, s):
    """PTX prmt in default mode: byte n of the result is byte (s >> 4n) & 7 of
    the eight bytes {x (bytes 0-3), y (bytes 4-7)}."""
    src = [(x >> (8 * i)) & 0xFF for i in range(4)] + [(y >> (8 * i)) & 0xFF for i in range(4)]
    return sum(src[(s >> (4 * n)) & 7] << (8 * n) for n in range(4))


def as_f32(bits):
    return struct.unpack("<f", struct.pack("<I", bits & 0xFFFFFFFF))[0]


def nib_bytes(w, hi):
    """Each byte of w becomes 0x80 | 8q for its low (hi=False) or high nibble q."""
    return ((((w >> 1) if hi else (w << 3)) & 0x78787878) | 0x80808080) & 0xFFFFFFFF


def nib16(v, i):
    """1 + q/16 for the nibble held in byte i of v: bits 0x3F800000 | q << 19."""
    return as_f32(byte_perm(v, 0x3F000000, 0x7044 | (i << 8)))


def test_nibble_decode_is_exact_for_every_byte():
    for byte in range(256):
        w = byte * 0x01010101  # the byte in every position
        for i in range(4):
            assert nib16(nib_bytes(w, False), i) == 1 + (byte & 15) / 16
            assert nib16(nib_bytes(w, True), i) == 1 + (byte >> 4) / 16


def test_block_dot_identity():
    """sum_e (q_e - 8) x_e = 16 sum_e f_e x_e - 24 sum_e x_e with f = 1 + q/16,
    and the down-phase form (16 h s) f - 24 h s = h s (q - 8)."""
    rng = np.random.default_rng(5)
    for _ in range(200):
        q = rng.integers(0, 16, 32)
        x = rng.standard_normal(32)
        f = 1 + q / 16
        assert np.isclose((q - 8) @ x, 16 * (f @ x) - 24 * x.sum(), rtol=0, atol=1e-12)
        hs = rng.standard_normal()
        np.testing.assert_allclose(16 * hs * f - 24 * hs, hs * (q - 8), rtol=0, atol=1e-12)


def test_block_bytes_map_to_elements():
    """Byte j of the 16 quant bytes holds element j (low nibble) and element
    j + 16 (high nibble); the decode walks words k = 0..3, bytes i = 0..3."""
    rng = np.random.default_rng(6)
    elems = rng.integers(0, 16, 32)
    qbytes = [int(elems[j]) | (int(elems[j + 16]) << 4) for j in range(16)]
    words = [sum(qbytes[4 * k + i] << (8 * i) for i in range(4)) for k in range(4)]
    got = [0] * 32
    for k in range(4):
        lo, hi = nib_bytes(words[k], False), nib_bytes(words[k], True)
        for i in range(4):
            got[4 * k + i] = round((nib16(lo, i) - 1) * 16)
            got[4 * k + i + 16] = round((nib16(hi, i) - 1) * 16)
    assert got == list(elems)


# ---------------------------------------------------------------------------
# permuted m16n8k16 fragments (batched row GEMM on tensor cores)
# ---------------------------------------------------------------------------
def mma_m16n8k16(a_regs, b_regs):
    """D = A B from per-lane fragments, following the documented operand layout
    of mma.m16n8k16 with 16-bit A (row) and B (col): lane = 4 g + t;
    A regs {0,1,2,3} hold A[g][2t..2t+1], A[g+8][2t..2t+1], A[g][2t+8..2t+9],
    A[g+8][2t+8..2t+9]; B regs {0,1} hold B[2t..2t+1][g], B[2t+8..2t+9][g];
    D element (row r, col c) is lane 4 (r % 8) + c // 2, value 2 (r // 8) + c % 2."""
    A = np.zeros((16, 16))
    Bm = np.zeros((16, 8))
    for lane in range(32):
        g, t = lane // 4, lane % 4
        a = a_regs[lane]
        for e in range(2):
            A[g][2 * t + e] = a[0][e]
            A[g + 8][2 * t + e] = a[1][e]
            A[g][2 * t + 8 + e] = a[2][e]
            A[g + 8][2 * t + 8 + e] = a[3][e]
            Bm[2 * t + e][g] = b_regs[lane][0][e]
            Bm[2 * t + 8 + e][g] = b_regs[lane][1][e]
    return A @ Bm


def test_permuted_fragments_cover_each_element_once():
    """Lane (g, t) loads elements [8t, 8t + 8) of a 32-element step as words
    W0..W3 (pairs); k-step 2s uses W0, W1 and k-step 2s+1 uses W2, W3."""
    seen = []
    for t in range(4):
        for word in range(4):
            for e in range(2):
                seen.append(8 * t + 2 * word + e)
    assert sorted(seen) == list(range(32))


@pytest.mark.parametrize("seed", range(5))
def test_permuted_fragments_give_the_plain_product(seed):
    rng = np.random.default_rng(seed)
    rows = rng.standard_normal((16, 32))   # 16 weight rows, one 32-element step
    toks = rng.standard_normal((8, 32))    # 8 tokens
    expect = rows @ toks.T                 # [16 rows x 8 tokens]
    acc = np.zeros((16, 8))
    for step in range(2):                  # k-steps 2s and 2s+1
        a_regs, b_regs = [], []
        for lane in range(32):
            g, t = lane // 4, lane % 4
            w = [[rows[g][8 * t + 2 * k + e] for e in range(2)] for k in range(4)]
            w8 = [[rows[g + 8][8 * t + 2 * k + e] for e in range(2)] for k in range(4)]
            x = [[toks[g][8 * t + 2 * k + e] for e in range(2)] for k in range(4)]
            lo = 2 * step  # words 0, 1 for step 2s; words 2, 3 for step 2s+1
            a_regs.append([w[lo], w8[lo], w[lo + 1], w8[lo + 1]])
            b_regs.append([x[lo], x[lo + 1]])
        acc += mma_m16n8k16(a_regs, b_regs)
    np.testing.assert_allclose(acc, expect, rtol=1e-12, atol=1e-12)
