"""The packed sign layout is the int8 tensor-core operand layout.

The decode kernels feed `word & (0x01010101 << q)` of a packed tile straight
to `mma.sync.aligned.m16n8k32` as the A operand (u8).  That is only right if,
for every lane and register, the four bytes of the word at bit position q hold
exactly the A elements that the PTX ISA assigns to that lane and register.
For the m16n8k32 A fragment of 8-bit types, the PTX ISA (section on the
matrix fragments of mma.m16n8k32) gives each lane (groupID g = lane / 4,
threadID_in_group c = lane % 4) four 32-bit registers a0..a3 of four bytes
each, byte i of register r holding
    row = g + 8 * (r % 2),    col = 4 * c + i + 16 * (r // 2).
This test restates that mapping and checks the oracle's layout against it:
bit 8*i + q of word r of lane L is element (row, col) of the q-th 16 x 32
operand block, for both roles.
"""
import numpy as np

from oracle import littlebit_oracle as orc


def _a_fragment(lane: int, r: int, i: int):
    g, c = lane // 4, lane % 4
    return g + 8 * (r % 2), 4 * c + i + 16 * (r // 2)


def test_role_v_planes_are_a_fragments_of_32_wide_k_blocks():
    row, k = orc._tile_coords("V", 1, 1)          # [rb, kt, lane, word, bit]
    for lane in range(32):
        for r in range(4):
            for n in range(32):
                i, q = n // 8, n % 8
                fr, fc = _a_fragment(lane, r, i)
                # plane q is the 16 x 32 block of latent rows 0..15 and inputs 32q..32q+31
                assert row[0, 0, lane, r, n] == fr
                assert k[0, 0, lane, r, n] == 32 * q + fc


def test_role_u_planes_are_a_fragments_of_16_row_blocks():
    row, k = orc._tile_coords("U", 1, 1)
    for lane in range(32):
        for r in range(4):
            for n in range(32):
                i, q = n // 8, n % 8
                fr, fc = _a_fragment(lane, r, i)
                # plane q is the 16 x 32 block of output rows 16q..16q+15 and latent 0..31
                assert row[0, 0, lane, r, n] == 16 * q + fr
                assert k[0, 0, lane, r, n] == fc


def test_masking_a_word_gives_the_plane_as_u8_values():
    """word & (0x01010101 << q): byte i is 2^q exactly when bit 8i+q is set,
    so the u8 operand is 2^q * [sign negative] and the product is 2^q times
    the plane's count, which the kernels shift back."""
    rng = np.random.default_rng(3)
    for _ in range(100):
        w = int(rng.integers(0, 2 ** 32))
        for q in range(8):
            m = w & (0x01010101 << q)
            for i in range(4):
                byte = (m >> (8 * i)) & 0xFF
                assert byte == ((w >> (8 * i + q)) & 1) << q
