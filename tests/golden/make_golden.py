"""Writes the hand-derived golden fixtures in this folder.

Every expected value here is worked out by hand from a closed form or from the
FP8 E4M3 / FP4 E2M1 format definitions; the script only records those values
as JSON.
It calls neither the CUDA library nor the oracle.

    python tests/golden/make_golden.py
"""

import json
import math
import os
import struct

HERE = os.path.dirname(os.path.abspath(__file__))
NAN16 = 0x7FC0  # bf16 quiet NaN, fills slots that must never be read


def bf(x: float) -> int:
    """bf16 bit pattern of a float that bf16 represents exactly."""
    bits = struct.unpack(">I", struct.pack(">f", x))[0]
    assert bits & 0xFFFF == 0, x
    return bits >> 16


def fixtures():
    g = {}
    g["two_keys"] = {
        "source": "closed form: softmax of the two scores 0 and ln 3 gives weights "
                  "1/4 and 3/4; lse = ln(1 + 3) = ln 4",
        "batch": 1, "q_len": 1, "num_q_heads": 1, "num_kv_heads": 1,
        "head_dim": 2, "page_size": 2, "kv_dtype": 0, "scale": "float32(ln 3)",
        "causal_offset": -1, "window": 0,
        "q_bits": [[[[bf(1.0), bf(0.0)]]]],
        "k_pages_bits": [[[[bf(0.0), bf(0.0)], [bf(1.0), bf(0.0)]]]],
        "v_pages_bits": [[[[bf(1.0), bf(0.0)], [bf(0.0), bf(1.0)]]]],
        "page_table": [[0]], "kv_lens": [2],
        "expected_out": [[[[0.25, 0.75]]]],
        "expected_lse": [[[math.log(4.0)]]],
        "tolerance": 1e-7,
        "note": "scale is ln 3 rounded to float32, so the values hold to ~1e-8",
    }

    # Bottom-right causal, q_len 2, window 3, kv_len 6, page size 4, page
    # table [1, 0]. Keys are zero, so every visible score is 0: out is the
    # mean of the visible v and lse = ln(count). v_j = [j, 1].
    # Row 0 sits at position 4 and sees keys {2, 3, 4}: out [3, 1].
    # Row 1 sits at position 5 and sees keys {3, 4, 5}: out [4, 1].
    table = [1, 0]
    kp = [[[[NAN16, NAN16] for _ in range(4)]] for _ in range(2)]
    vp = [[[[NAN16, NAN16] for _ in range(4)]] for _ in range(2)]
    for j in range(6):
        pg, r = table[j // 4], j % 4
        kp[pg][0][r] = [bf(0.0), bf(0.0)]
        vp[pg][0][r] = [bf(float(j)), bf(1.0)]
    g["window_causal_equal_keys"] = {
        "source": "closed form: equal keys give uniform weights, so out is the mean "
                  "of the visible v and lse = ln |visible set|; visible sets "
                  "enumerated by hand (bottom-right rows, window of 3 keys that "
                  "includes the query)",
        "batch": 1, "q_len": 2, "num_q_heads": 1, "num_kv_heads": 1,
        "head_dim": 2, "page_size": 4, "kv_dtype": 0, "scale": 0.5,
        "causal_offset": -2, "window": 3,
        "q_bits": [[[[bf(0.75), bf(-1.5)]], [[bf(2.0), bf(1.0)]]]],
        "k_pages_bits": kp, "v_pages_bits": vp,
        "page_table": [table], "kv_lens": [6],
        "expected_out": [[[[3.0, 1.0]], [[4.0, 1.0]]]],
        "expected_lse": [[[math.log(3.0)], [math.log(3.0)]]],
        "tolerance": 1e-12,
    }

    # GQA: Hq 4, Hkv 2, one key per kv head. kv head 0: k [1, 0], v [10, 20];
    # kv head 1: k [0, 1], v [-3, 5]. Every q head is [1, 2], scale 0.25:
    # heads 0, 1 score 0.25; heads 2, 3 score 0.5.
    g["gqa_single_key"] = {
        "source": "closed form: one visible key has weight 1, so out = v and "
                  "lse = scale * q.k; heads 0, 1 read kv head 0 and heads 2, 3 "
                  "read kv head 1 (consecutive grouping)",
        "batch": 1, "q_len": 1, "num_q_heads": 4, "num_kv_heads": 2,
        "head_dim": 2, "page_size": 1, "kv_dtype": 0, "scale": 0.25,
        "causal_offset": -1, "window": 0,
        "q_bits": [[[[bf(1.0), bf(2.0)]] * 4]],
        "k_pages_bits": [[[[bf(1.0), bf(0.0)]], [[bf(0.0), bf(1.0)]]]],
        "v_pages_bits": [[[[bf(10.0), bf(20.0)]], [[bf(-3.0), bf(5.0)]]]],
        "page_table": [[0]], "kv_lens": [1],
        "expected_out": [[[[10.0, 20.0], [10.0, 20.0], [-3.0, 5.0], [-3.0, 5.0]]]],
        "expected_lse": [[[0.25, 0.25, 0.5, 0.5]]],
        "tolerance": 1e-12,
    }

    g["empty_row"] = {
        "source": "definition: a row with no visible key has out = 0 and lse = -inf; "
                  "a single key gives out = v and lse = scale * q.k = 1",
        "batch": 2, "q_len": 1, "num_q_heads": 1, "num_kv_heads": 1,
        "head_dim": 2, "page_size": 2, "kv_dtype": 0, "scale": 1.0,
        "causal_offset": -1, "window": 0,
        "q_bits": [[[[bf(1.0), bf(1.0)]]], [[[bf(1.0), bf(1.0)]]]],
        "k_pages_bits": [[[[bf(1.0), bf(0.0)], [NAN16, NAN16]]]],
        "v_pages_bits": [[[[bf(7.0), bf(-7.0)], [NAN16, NAN16]]]],
        "page_table": [[0], [-1]], "kv_lens": [1, 0],
        "expected_out": [[[[7.0, -7.0]]], [[[0.0, 0.0]]]],
        "expected_lse": [[[1.0]], [["-inf"]]],
        "tolerance": 1e-12,
    }

    g["e4m3_codes"] = {
        "source": "OCP 8-bit floating point, E4M3: (-1)^s * 2^(e-7) * (1 + m/8); "
                  "exponent 0 is subnormal 2^-6 * m/8; no infinities; S.1111.111 "
                  "is NaN; largest finite 448. Values worked by hand.",
        "codes": [0x00, 0x80, 0x01, 0x07, 0x08, 0x38, 0x3C, 0x40, 0xC0, 0x7E,
                  0xFE, 0x7F, 0xFF, 0x77, 0x30],
        "values": [0.0, -0.0, 0.001953125, 0.013671875, 0.015625, 1.0, 1.5, 2.0,
                   -2.0, 448.0, -448.0, "nan", "nan", 240.0, 0.5],
    }
    g["e2m1_codes"] = {
        "source": "OCP FP4 E2M1: (-1)^s * 2^(e-1) * (1 + m/2) for exponent field e "
                  "in 1..3; exponent 0 is subnormal m/2; no infinities or NaN; "
                  "largest magnitude 6. Code bits s e1 e0 m. Values worked by hand.",
        "codes": list(range(16)),
        "values": [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,
                   -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0],
    }
    g["nvfp4_blocks"] = {
        "source": "NVFP4 block quantisation worked by hand: q = x / kv_scale; "
                  "scale = e4m3(max|q| / 6) to nearest (ties even, saturating at "
                  "448); code = e2m1(q / scale) to nearest, ties to the even "
                  "mantissa bit, saturating at 6, sign kept; a zero scale stores "
                  "+0 codes. Block 1: max|q| = 7, 7/6 = 1.1667 is nearest the "
                  "e4m3 value 1.125 (code 0x39); q/1.125 gives 6.22 -> 6, 0.889 -> 1, "
                  "2.5 -> 2 (tie, even), -0.222 -> -0, 0, -0, 0.5, 3.5 -> 4 (tie), "
                  "-6.22 -> -6, 0.111 -> 0, 1.5, 4, -5 -> -4 (tie), 0.25 -> 0 (tie), "
                  "2, -1.25 -> -1 (tie). Block 2: all zero, scale code 0, codes +0. "
                  "Block 3: kv_scale 0.5, q = 6, -3, 1, 0 ... -> scale 1 (0x38). "
                  "Block 4: kv_scale 2^-10, q = 2^22 -> scale saturates at 448 "
                  "(0x7E), codes saturate at 6.",
        "blocks": [
            {"kv_scale": 1.0,
             "x_bits": [bf(v) for v in (7.0, 1.0, 2.8125, -0.25, 0.0, -0.0, 0.5625,
                                        3.9375, -7.0, 0.125, 1.6875, 4.5, -5.625,
                                        0.28125, 2.25, -1.40625)],
             "scale_code": 0x39,
             "codes": [0x7, 0x2, 0x4, 0x8, 0x0, 0x8, 0x1, 0x6, 0xF, 0x0, 0x3, 0x6,
                       0xE, 0x0, 0x4, 0xA]},
            {"kv_scale": 1.0,
             "x_bits": [bf(v) for v in (0.0, -0.0) * 8],
             "scale_code": 0x00, "codes": [0x0] * 16},
            {"kv_scale": 0.5,
             "x_bits": [bf(v) for v in (3.0, -1.5, 0.5, 0.0) * 4],
             "scale_code": 0x38, "codes": [0x7, 0xD, 0x2, 0x0] * 4},
            {"kv_scale": 2.0 ** -10,
             "x_bits": [bf(v) for v in (4096.0, -4096.0, 1.0, 0.0) * 4],
             "scale_code": 0x7E, "codes": [0x7, 0xF, 0x4, 0x0] * 4},
        ],
    }
    return g


if __name__ == "__main__":
    for name, obj in fixtures().items():
        with open(os.path.join(HERE, f"{name}.json"), "w") as f:
            json.dump(obj, f, indent=1)
