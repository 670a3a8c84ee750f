"""Write the hand-built quantised-block fixtures of this folder.

    python tests/golden/make_golden.py           # rewrite the JSON files
    python tests/golden/make_golden.py --check   # exit 1 if a file differs

Each fixture entry is chosen by hand: a name, the fp16 scale bits and the 32
codes.  This script only packs them into the canonical block bytes of each
format with Python's `struct` and integer operations; it imports nothing
from the oracle or from the CUDA package, so the fixtures pin the oracle's
decoders from the outside.  The layouts (the source pages name the formats
but print no layout; the canonical llama.cpp blocks are the reading taken):

  Q4_0  2-byte little-endian fp16 scale, then 16 bytes; byte j holds code j
        in its low nibble and code j+16 in its high nibble; weight d*(q-8).
  Q8_0  2-byte scale, then 32 signed bytes, element j in byte j; weight d*q.
  Q5_0  2-byte scale, a little-endian 32-bit word whose bit j is the fifth
        bit of element j, then 16 bytes of low nibbles as in Q4_0;
        weight d*(q-16).
  q6_K  super-blocks of 256 weights in 210 bytes: ql[128], qh[64], 16
        signed 8-bit sub-block scales, then the 2-byte fp16 scale d.  Element
        i = 128 h + 32 c + l takes its low 4 bits from the low (c < 2) or high
        (c >= 2) nibble of ql[64 h + 32 (c % 2) + l] and its high 2 bits from
        bits 2c, 2c+1 of qh[32 h + l]; weight d * sc[i // 16] * (q - 32).
"""
from __future__ import annotations

import json
import os
import struct
import sys

HERE = os.path.dirname(os.path.abspath(__file__))

ABOUT = {
    "q4_0": (
        "Hand-built canonical Q4_0 blocks. Source of the format: the weight-format statement "
        "that each block holds an fp16 scale d plus 32 4-bit codes q in 0..15 along the "
        "reduction dimension, with weight = d*(q-8) (35B-A3B Q4_0 workload); the 'MoE on RTX "
        "5090 reaches 41% of bandwidth' page names Q4_0 as the quantisation (measurement-setup "
        "paragraph) and the MMVQ page says quantised weights are read once and never expanded "
        "(section on MMVQ). Byte order (our reading, the canonical llama.cpp one): 2 bytes "
        "little-endian fp16 scale, then 16 bytes where byte j holds code j in its low nibble "
        "and code j+16 in its high nibble. Each entry lists the 18 bytes and, separately, the "
        "32 codes and the scale bits they were built from; the expected weights are "
        "scale*(code-8)."),
    "q8_0": (
        "Hand-built canonical Q8_0 blocks. The 'MoE on RTX 5090 reaches 41% of bandwidth' page "
        "names q8_0 among the quantisation formats of the 35B-A3B model it measures (the "
        "paragraph on the model's mix of formats) but prints no layout; our reading is the "
        "canonical llama.cpp block: 2 bytes little-endian fp16 scale d, then 32 signed bytes "
        "(two's complement), element j in byte j; weight = d*q. Each entry lists the 34 bytes "
        "and, separately, the 32 codes and the scale bits they were built from; the expected "
        "weights are scale*code."),
    "q5_0": (
        "Hand-built canonical Q5_0 blocks. The 'MoE on RTX 5090 reaches 41% of bandwidth' page "
        "names q5_0 among the quantisation formats of the 35B-A3B model it measures "
        "(measurement-setup paragraph) but prints no layout; our reading is the canonical "
        "llama.cpp block: 2 bytes little-endian fp16 scale d, a little-endian 32-bit word qh "
        "whose bit j is the fifth bit of element j, then 16 bytes where byte j holds the low 4 "
        "bits of element j (low nibble) and of element j+16 (high nibble); weight = d*(q-16) "
        "with q = low bits + 16 * fifth bit. Each entry lists the 22 bytes and, separately, "
        "the 32 codes and the scale bits they were built from; the expected weights are "
        "scale*(code-16)."),
}

# (name, fp16 scale bits, 32 codes), chosen by hand: ramps, extremes, the
# smallest subnormal and the largest normal scale, a negative scale.
SPECS = {
    "q4_0": [
        ("ramp, scale 0.5", 0x3800, list(range(16)) + list(range(15, -1, -1))),
        ("smallest subnormal scale, all codes 0", 0x0001, [0] * 32),
        ("negative scale -2, all codes 8 (all weights zero)", 0xC000, [8] * 32),
        ("largest normal scale 65504, code 15 at element 0 and code 1 at element 31", 0x7BFF,
         [15] + [8] * 30 + [1]),
    ],
    "q8_0": [
        ("ramp -16..15, scale 1", 0x3C00, list(range(-16, 16))),
        ("extremes -128 and 127 alternating, scale 0.5", 0x3800, [-128, 127] * 16),
        ("negative scale -2, codes -1, 0, 1 repeated", 0xC000, ([-1, 0, 1] * 11)[:32]),
        ("smallest subnormal scale, all codes -128", 0x0001, [-128] * 32),
        ("largest normal scale 65504, code 127 at element 0 and -128 at element 31", 0x7BFF,
         [127] + [0] * 30 + [-128]),
    ],
    "q5_0": [
        ("ramp 0..31 (weights -16..15), scale 1", 0x3C00, list(range(32))),
        ("descending 31..0, scale 0.5", 0x3800, list(range(31, -1, -1))),
        ("alternating 16 / 15 (weights 0 / -1), scale -2", 0xC000, [16, 15] * 16),
        ("smallest subnormal scale, all codes 31", 0x0001, [31] * 32),
        ("largest normal scale 65504, code 0 at element 0 and 31 at element 31, 16 elsewhere",
         0x7BFF, [0] + [16] * 30 + [31]),
    ],
}


def pack_q4_0(scale_bits: int, codes) -> bytes:
    assert len(codes) == 32 and all(0 <= q < 16 for q in codes)
    qs = bytes(codes[j] | (codes[j + 16] << 4) for j in range(16))
    return struct.pack("<H", scale_bits) + qs


def pack_q8_0(scale_bits: int, codes) -> bytes:
    assert len(codes) == 32 and all(-128 <= q < 128 for q in codes)
    return struct.pack("<H32b", scale_bits, *codes)


def pack_q5_0(scale_bits: int, codes) -> bytes:
    assert len(codes) == 32 and all(0 <= q < 32 for q in codes)
    qh = 0
    for j, q in enumerate(codes):
        qh |= (q >> 4) << j
    qs = bytes((codes[j] & 15) | ((codes[j + 16] & 15) << 4) for j in range(16))
    return struct.pack("<HI", scale_bits, qh) + qs


PACK = {"q4_0": pack_q4_0, "q8_0": pack_q8_0, "q5_0": pack_q5_0}

ABOUT["q6_k"] = (
    "Hand-built canonical q6_K super-blocks. The 'MoE on RTX 5090 reaches 41% of bandwidth' "
    "page names q6_K among the quantisation formats of the 35B-A3B model it measures "
    "(measurement-setup paragraph) but prints no layout; our reading is the canonical "
    "llama.cpp super-block of 256 weights in 210 bytes: ql[128] (low 4 bits), qh[64] (high 2 "
    "bits), 16 signed 8-bit sub-block scales, then a little-endian fp16 super-block scale d. "
    "Element i = 128h + 32c + l takes its low 4 bits from the low (c < 2) or high (c >= 2) "
    "nibble of ql[64h + 32(c%2) + l] and its high 2 bits from bits 2c, 2c+1 of qh[32h + l]; "
    "weight = d * sc[i/16] * (q - 32). Each entry lists the 210 bytes and, separately, the "
    "256 codes, the 16 sub-scales and the scale bits they were built from.")

# (name, fp16 scale bits, 16 sub-scales, 256 codes)
SPECS_Q6K = [
    ("ramp 0..63 four times, sub-scales 1..16, scale 1", 0x3C00, list(range(1, 17)),
     [i % 64 for i in range(256)]),
    ("codes 0 / 63 alternating, sub-scales -128 / 127 alternating, scale 0.5", 0x3800,
     [-128, 127] * 8, [0, 63] * 128),
    ("smallest subnormal scale, all codes 63, sub-scales -1", 0x0001, [-1] * 16, [63] * 256),
    ("largest normal scale 65504, code 63 at element 0 and 0 at element 255, 32 elsewhere, "
     "sub-scales 1", 0x7BFF, [1] * 16, [63] + [32] * 254 + [0]),
    ("scrambled codes (37 i mod 64), sub-scales j - 8, scale -0.25", 0xB400,
     [j - 8 for j in range(16)], [(37 * i) % 64 for i in range(256)]),
]


def pack_q6_k(scale_bits: int, sub_scales, codes) -> bytes:
    assert len(codes) == 256 and all(0 <= q < 64 for q in codes)
    assert len(sub_scales) == 16 and all(-128 <= s < 128 for s in sub_scales)
    ql = [0] * 128
    qh = [0] * 64
    for i, q in enumerate(codes):
        h, r = divmod(i, 128)
        c, l = divmod(r, 32)
        j = 64 * h + 32 * (c % 2) + l
        ql[j] |= (q & 15) << (4 if c >= 2 else 0)
        qh[32 * h + l] |= (q >> 4) << (2 * c)
    return bytes(ql) + bytes(qh) + struct.pack("<16b", *sub_scales) + struct.pack("<H", scale_bits)


def fixture(fmt: str) -> dict:
    if fmt == "q6_k":
        blocks = [{"name": name, "bytes": list(pack_q6_k(sb, scs, codes)), "scale_bits": sb,
                   "sub_scales": list(scs), "codes": list(codes)}
                  for name, sb, scs, codes in SPECS_Q6K]
        return {"about": ABOUT[fmt], "blocks": blocks}
    blocks = [{"name": name, "bytes": list(PACK[fmt](sb, codes)), "scale_bits": sb,
               "codes": list(codes)} for name, sb, codes in SPECS[fmt]]
    return {"about": ABOUT[fmt], "blocks": blocks}


def text(fmt: str) -> str:
    return json.dumps(fixture(fmt), indent=1)


def main(argv) -> int:
    check = "--check" in argv
    bad = 0
    for fmt in list(SPECS) + ["q6_k"]:
        path = os.path.join(HERE, f"{fmt}_blocks.json")
        want = text(fmt)
        if check:
            with open(path) as f:
                if json.load(f) != json.loads(want):
                    print(f"{path}: differs from what this script writes")
                    bad = 1
        else:
            with open(path, "w") as f:
                f.write(want)
    return bad


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
