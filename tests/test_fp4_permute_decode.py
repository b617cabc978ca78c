"""The FP4 tensor-core decode turns E2M1 codes into bf16 with byte permutes
(`prmt.b32`) on two 8-byte tables instead of a lookup in shared memory. This
host test reads the table constants and selectors out of the kernel source,
applies them with the PTX definition of `prmt` (default mode: selector bits
0-2 pick one of the eight bytes {b, a}, bit 3 replicates that byte's sign bit),
and checks every 32-bit code word pattern class against the oracle's E2M1
value table: all 256 code bytes in each of the four byte positions, plus
random words. Bit-exact, including the sign of zero.
"""
import os
import re
import struct

import numpy as np

from oracle import v41

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "latent_kv_decode_b200", "csrc", "decode_fp4_sm100.cu")


def _prmt(a: int, b: int, sel: int) -> int:
    src = [(a >> (8 * i)) & 0xFF for i in range(4)] + [(b >> (8 * i)) & 0xFF for i in range(4)]
    out = 0
    for n in range(4):
        s = (sel >> (4 * n)) & 0xF
        byte = src[s & 7]
        if s & 8:
            byte = 0xFF if byte & 0x80 else 0x00
        out |= byte << (8 * n)
    return out


def _kernel_constants():
    body = open(SRC).read()
    fn = body[body.index("e2m1x8_to_bf16x2(uint32_t x"):]
    fn = fn[:fn.index("\n}\n")]
    c = {k: int(v, 16) for k, v in re.findall(r"(k(?:Lo|Hi)\d\d) = 0x([0-9A-Fa-f]+)u", fn)}
    sign_hi, sign_lo = (int(v, 16) for v in re.search(r"h \? 0x([0-9A-Fa-f]+)u : 0x([0-9A-Fa-f]+)u", fn).groups())
    inter = [int(v, 16) for v in re.findall(r"prmt\(lo, hi, 0x([0-9A-Fa-f]+)u\)", fn)]
    mag_mask = int(re.search(r"& 0x([0-9A-Fa-f]+)u;\n", fn).group(1), 16)
    sign_mask = int(re.search(r"\(sg & 0x([0-9A-Fa-f]+)u\)", fn).group(1), 16)
    return c, sign_lo, sign_hi, inter, mag_mask, sign_mask


def _decode_word(x: int, k):
    c, sign_lo, sign_hi, inter, mag_mask, sign_mask = k
    x4 = (x << 4) & 0xFFFFFFFF
    w = []
    for h in range(2):
        sel = ((x >> 16) if h else x) & mag_mask
        lo = _prmt(c["kLo03"], c["kLo47"], sel)
        sg = _prmt(x4, x, sign_hi if h else sign_lo)
        hi = _prmt(c["kHi03"], c["kHi47"], sel) | (sg & sign_mask)
        w += [_prmt(lo, hi, inter[0]), _prmt(lo, hi, inter[1])]
    return w


def _bf16(h: int) -> float:
    return struct.unpack("<f", struct.pack("<I", h << 16))[0]


def test_permute_decode_matches_e2m1_table_bit_exactly():
    k = _kernel_constants()
    assert len(k[3]) == 2
    rng = np.random.Generator(np.random.PCG64(3))
    words = [int(v) << (8 * pos) for pos in range(4) for v in range(256)]
    words += [int(v) for v in rng.integers(0, 2**32, 2000, dtype=np.uint64)]
    for x in words:
        w = _decode_word(x, k)
        codes = np.array([(x >> (4 * i)) & 0xF for i in range(8)], np.uint8)
        want = v41.e2m1_decode(codes)
        for i in range(8):
            got = _bf16((w[i // 2] >> (16 * (i % 2))) & 0xFFFF)
            assert got == want[i] and np.signbit(got) == np.signbit(want[i]), (hex(x), i, got, want[i])
