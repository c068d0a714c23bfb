"""The fp64 oracle against its pins (CPU only)."""

import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import oracle as orc
from paged_kv_decode_30_b200 import workloads as W
from tests import oracle_pins as pins


@pytest.fixture(scope="module")
def lib():
    return orc.load()


def test_bf16_decode_matches_torch(lib):
    pins.check_decode_bf16(lib)


def test_e4m3_decode_matches_torch_and_format(lib):
    pins.check_decode_e4m3(lib)


@pytest.mark.parametrize("name", pins.GOLDEN_NAMES)
def test_golden(lib, name):
    pins.check_golden(name, lib)


@pytest.mark.parametrize("wl", pins.SMALL_CASES, ids=lambda w: w.name)
def test_bruteforce_dense_attention(lib, wl):
    pins.check_bruteforce(wl, lib)


@pytest.mark.parametrize("wl", pins.SMALL_CASES[:4] + pins.SMALL_CASES[6:7], ids=lambda w: w.name)
def test_page_permutation_is_bit_identical(lib, wl):
    pins.check_page_permutation(wl, lib)


@pytest.mark.parametrize("cuts", [[1], [37], [64, 65], [16, 48, 96], [0, 500]])
def test_split_merge_equals_unsplit(lib, cuts):
    pins.check_split_merge(pins.SMALL_CASES[3], cuts, lib)
    pins.check_split_merge(pins.SMALL_CASES[6], cuts, lib)


def test_equal_keys_mean_of_values(lib):
    pins.check_equal_keys(lib)


def test_one_hot_values_give_probabilities(lib):
    pins.check_one_hot_values(lib)


@pytest.mark.parametrize("wl", [pins.SMALL_CASES[0], pins.SMALL_CASES[3],
                                pins.SMALL_CASES[5], pins.SMALL_CASES[6]],
                         ids=lambda w: w.name)
def test_poisoned_slots_are_never_read(lib, wl):
    pins.check_poison_is_never_read(wl, lib)


def test_single_key_returns_value(lib):
    wl = W.Workload(name="single", batch=3, num_q_heads=4, num_kv_heads=2,
                    head_dim=16, page_size=4, kv_lens=("fixed", [1, 1, 1]),
                    route="dense", seed=31)
    inp = W.generate(wl)
    out, lse = pins.run_oracle(inp, lib)
    q = inp["q"].double().numpy()
    for b in range(3):
        V = inp["v_dense"][b].double().numpy()
        K = inp["k_dense"][b].double().numpy()
        for h in range(4):
            g = h // 2
            np.testing.assert_array_equal(out[b, 0, h], V[g, 0])
            s = W.scale_of(wl) * float(q[b, 0, h] @ K[g, 0])
            assert abs(lse[b, 0, h] - s) <= 1e-12


def test_merge_single_state_is_identity(lib):
    rng = np.random.default_rng(0)
    o = rng.standard_normal((1, 5, 8))
    ls = rng.standard_normal((1, 5))
    mo, ml = orc.merge_states(o, ls, lib=lib)
    pins.assert_close(mo, o[0], 1e-15, "identity out")
    pins.assert_close(ml, ls[0], 1e-15, "identity lse")


def test_merge_ignores_empty_states(lib):
    rng = np.random.default_rng(1)
    o = rng.standard_normal((3, 4, 8))
    ls = rng.standard_normal((3, 4))
    ls[1] = -np.inf
    o[1] = np.nan  # an empty state's output must never be read
    mo, ml = orc.merge_states(o, ls, lib=lib)
    ref_o, ref_l = orc.merge_states(o[[0, 2]], ls[[0, 2]], lib=lib)
    np.testing.assert_array_equal(mo, ref_o)
    np.testing.assert_array_equal(ml, ref_l)
    ls[:] = -np.inf
    mo, ml = orc.merge_states(o, ls, lib=lib)
    assert (mo == 0).all() and np.isneginf(ml).all()


def test_workload_recipes_match_stated_shapes():
    """The generator's large recipes produce the stated sizes (host only)."""
    import torch
    gen = torch.Generator().manual_seed(W.VARLEN.seed)
    lens = W._draw_kv_lens(W.VARLEN, gen)
    assert lens.min() >= 512 and lens.max() <= 4096 and lens.numel() == 32
    lens = W._draw_kv_lens(W.FP8_VERIFY, torch.Generator().manual_seed(W.FP8_VERIFY.seed))
    assert lens.min() >= 128 and lens.max() <= 32768 and lens.numel() == 64
    assert W.visible_token_count(W.HEADLINE, [8192] * 128) == 128 * 8192
    # bottom-right rows with a window of 4096 see at most 4096 + 3 keys
    assert W.visible_token_count(W.FP8_VERIFY, [10000]) == 4099
    assert W.visible_token_count(W.FP8_VERIFY, [100]) == 100


# --------------------------------------------------------------------------
# Planted mistakes: each mutated copy of the oracle must fail the pins.

MUTATIONS = {
    "gqa_mapping": ("const int g = h / G;", "const int g = h % Hkv;"),
    "window_off_by_one": ("pos - (int64_t)window + 1", "pos - (int64_t)window"),
    "causal_strict": ("if (causal && j > pos) return 0;", "if (causal && j >= pos) return 0;"),
    "lse_drops_max": ("const double row_lse = m + log(sum);", "const double row_lse = log(sum);"),
    "page_row_swapped": ("const int64_t row = j % page_size;", "const int64_t row = j / page_size;"),
    "scale_dropped": ("s[j] = dscale * dot;", "s[j] = dot;"),
    "e4m3_bias": ("mag = ldexp(1.0 + (double)m / 8.0, e - 7);",
                  "mag = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "merge_weight": ("const double w = exp(ls - total);", "const double w = exp(ls - m);"),
    "bottom_right_shift": ("return kv_len - (int64_t)q_len + i;", "return kv_len - (int64_t)q_len + i - 1;"),
    "kv_scale_dropped": ("* kv_scale;\n}", ";\n}"),
    "e4m3_ties_to_odd": ("(c & 1) == 0 && (best & 1) == 1", "(c & 1) == 1 && (best & 1) == 0"),
    "append_slot_shifted": ("+ pos % page_size) * D;", "+ (pos + 1) % page_size) * D;"),
    "append_scale_inverted": ("oracle_e4m3_encode(kx / kv_scale)", "oracle_e4m3_encode(kx * kv_scale)"),
    "sink_dropped": ("if (sink != -INFINITY) sum += exp(sink - m);", ""),
    "sink_empty_row": ("*lrow = sink;", "*lrow = -INFINITY;"),
    "quantize_q_scale_off_by_one": ("const int e = mx > 0.0 ? 7 - ilogb(mx) : 0;",
                                    "const int e = mx > 0.0 ? 8 - ilogb(mx) : 0;"),
    "e2m1_bias": ("mag = ldexp(1.0 + (double)m / 2.0, e - 1);",
                  "mag = ldexp(1.0 + (double)m / 2.0, e - 2);"),
    "nvfp4_nibble_order": ("(index % 2) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF)",
                           "(index % 2) ? (uint8_t)(byte & 0xF) : (uint8_t)(byte >> 4)"),
    "nvfp4_block_index": ("((const uint8_t*)scales)[index / 16]",
                          "((const uint8_t*)scales)[index / 32]"),
    "nvfp4_block_scale_dropped": ("return oracle_e2m1_to_double(code) * block * kv_scale;",
                                  "return oracle_e2m1_to_double(code) * kv_scale;"),
    "e2m1_ties_to_odd": ("(best & 1) == 1 && (c & 1) == 0", "(best & 1) == 0 && (c & 1) == 1"),
    "nvfp4_amax_over_4": ("oracle_e4m3_encode(amax / 6.0f)", "oracle_e4m3_encode(amax / 4.0f)"),
    "nvfp4_zero_scale_keeps_sign": ("sd > 0.f ? oracle_e2m1_encode(q[d] / sd) : 0;",
                                    "sd > 0.f ? oracle_e2m1_encode(q[d] / sd) : (signbit(q[d]) ? 8 : 0);"),
    "nvfp4_append_nibbles_swapped": ("(uint8_t)(c[d] | (c[d + 1] << 4))",
                                     "(uint8_t)(c[d + 1] | (c[d] << 4))"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, name):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    src = open(orc._SRC).read()
    old, new = MUTATIONS[name]
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new)
    c = tmp_path / "oracle_mut.c"
    c.write_text(mutated)
    so = tmp_path / "liboracle_mut.so"
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fPIC", "-shared",
                    str(c), "-o", str(so), "-lm"], check=True)
    mlib = orc.load(str(so))
    with pytest.raises(AssertionError):
        pins.run_all(mlib)


@pytest.mark.parametrize("wl", [pins.SMALL_CASES[3], pins.SMALL_CASES[6]], ids=lambda w: w.name)
def test_multithreaded_oracle_is_bit_identical(lib, wl):
    """The OpenMP entry point (used to time the oracle on all host cores)
    runs the single-threaded row routine per row: identical bits."""
    inp = W.generate(wl, device="cpu")
    ref = pins.run_oracle(inp, lib)
    got = pins.run_oracle(inp, lib, threads=4)
    assert np.array_equal(ref[0], got[0]) and np.array_equal(ref[1], got[1])


def test_e4m3_encode_inverts_decode(lib):
    pins.check_e4m3_encode_roundtrip(lib)


def test_e4m3_encode_matches_torch_cast(lib):
    pins.check_e4m3_encode_vs_torch(lib)


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8_E4M3, W.KV_NVFP4])
def test_append_places_rows_by_page_table(lib, kv_dtype):
    pins.check_append(lib, kv_dtype)


def test_e2m1_decode_matches_ml_dtypes_and_format(lib):
    pins.check_decode_e2m1(lib)


def test_e2m1_encode_matches_ml_dtypes_cast(lib):
    pins.check_e2m1_encode_vs_ml_dtypes(lib)


def test_nvfp4_block_quantiser_hand_worked(lib):
    pins.check_nvfp4_block_golden(lib)


def test_nvfp4_block_quantiser_matches_restatement(lib):
    pins.check_nvfp4_block_vs_restated(lib)


@pytest.mark.parametrize("wl", pins.NVFP4_CASES, ids=lambda w: w.name)
def test_nvfp4_poisoned_scales_are_never_read(lib, wl):
    pins.check_poison_is_never_read(wl, lib)


def test_nvfp4_multithreaded_oracle_is_bit_identical(lib):
    inp = W.generate(pins.NVFP4_CASES[0], device="cpu")
    ref = pins.run_oracle(inp, lib)
    got = pins.run_oracle(inp, lib, threads=4)
    assert np.array_equal(ref[0], got[0]) and np.array_equal(ref[1], got[1])


@pytest.mark.parametrize("wl", [pins.SMALL_CASES[i] for i in (0, 2, 3, 6, 7, 8)], ids=lambda w: w.name)
def test_sink_matches_bruteforce_with_a_zero_value_key(lib, wl):
    pins.check_sink_bruteforce(wl, lib)


def test_sink_of_minus_infinity_changes_nothing(lib):
    pins.check_sink_neg_inf_is_no_sink(pins.SMALL_CASES[3], lib)


def test_native_qk_quantisation_matches_torch(lib):
    pins.check_quantize_q_vs_torch(lib)
