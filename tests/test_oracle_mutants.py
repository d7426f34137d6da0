"""Plants plausible mistakes in a copy of the oracle's C source and checks that a named
pin catches each one.  The mistakes live here, in the test, never in the oracle: each
mutant is compiled into a temporary library, the pin runs against it, and the pin must
fail.  This shows the pins are sensitive to a dropped term, a wrong sign, index or
operand anywhere in the oracle."""
import os

import pytest

import oracle
import tests.test_oracle_pins as pins

SRC = open(os.path.join(os.path.dirname(oracle.__file__), "pkv_oracle.c")).read()


def _golden():
    from tests.conftest import GOLDEN
    import json

    def load(name):
        with open(os.path.join(GOLDEN, name)) as f:
            return json.load(f)
    return load


# (name, text in the oracle, planted replacement, pin expected to catch it)
MUTANTS = [
    ("dropped_last_dim", "acc += qrow[j] * pool_value(k_pool", "if (j + 1 < d) acc += qrow[j] * pool_value(k_pool",
     lambda: pins.test_decode_equals_contiguous_attention(2)),
    ("softmax_sign", "double w = exp(s_buf[t] - m);", "double w = exp(m - s_buf[t]);",
     lambda: pins.test_closed_forms()),
    ("scale_dropped", "s_buf[t] = scale * acc;", "s_buf[t] = acc;",
     lambda: pins.test_decode_equals_contiguous_attention(3)),
    ("no_normalisation", "for (int j = 0; j < d; ++j) out[j] /= denom;", ";",
     lambda: pins.test_closed_forms()),
    ("values_from_k", "out[j] += w * pool_value(v_pool, v_scale", "out[j] += w * pool_value(k_pool, k_scale",
     lambda: pins.test_decode_equals_contiguous_attention(0)),
    ("gqa_interleaved", "qrow, h / G,\n                            block_tables",
     "qrow, h % H_kv,\n                            block_tables",
     lambda: pins.test_gqa_group_mapping_is_contiguous()),
    ("table_index", "int blk = table[t / ORC_BLOCK], off = t % ORC_BLOCK;\n        if (blk < 0",
     "int blk = table[t % ORC_BLOCK < 0 ? 0 : t / ORC_BLOCK / 2], off = t % ORC_BLOCK;\n        if (blk < 0",
     lambda: pins.test_block_table_figure(_golden())),
    ("window_off_by_one", "? n - window : 0;", "? n - window + 1 : 0;",
     lambda: pins.test_sliding_window_equals_library_attention_over_the_last_positions(5)),
    ("causal_off_by_one", "window), ctx_before + i + 1,", "window), ctx_before + i,",
     lambda: pins.test_prefill_chunk_rows_equal_decode_and_causal_library()),
    ("size_factor_two", "return (int64_t)2 * layers", "return (int64_t)layers",
     lambda: pins.test_bytes_per_token_worked_values(_golden())),
    ("round_half_away", "float c = rintf(r);", "float c = roundf(r);",
     lambda: pins.test_quant_golden_codes(_golden())),
    ("int4_levels", "case ORC_INT4: return 7.0;", "case ORC_INT4: return 8.0;",
     lambda: pins.test_quant_golden_codes(_golden())),
    ("int4_nibble_order", "int nib = (dd & 1) ? (byte >> 4) : (byte & 0xf);",
     "int nib = (dd & 1) ? (byte & 0xf) : (byte >> 4);",
     lambda: pins.test_quant_golden_codes(_golden())),
    ("e4m3_ties_away", "double m = nearbyint((2.0 * fr - 1.0) * 8.0);", "double m = round((2.0 * fr - 1.0) * 8.0);",
     lambda: pins.test_e4m3_golden_and_exhaustive(_golden())),
    ("e4m3_bias", "v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 8);",
     lambda: pins.test_e4m3_golden_and_exhaustive(_golden())),
    ("no_requantize", "if (s > s_old && s_old > 0.0f) {", "if (0) {",
     lambda: pins.test_quant_incremental_appends(oracle.INT8)),
    ("never_fresh", "float s_old = fresh ? 0.0f : scales[si];", "float s_old = scales[si];",
     lambda: pins.test_quant_block_reuse_starts_fresh(oracle.INT8)),
    ("scale_shrinks", "float s = s_old > a_over_q ? s_old : a_over_q;", "float s = a_over_q;",
     lambda: pins.test_quant_incremental_appends(oracle.INT4)),
]


@pytest.mark.parametrize("name,old,new,pin", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pin_catches_planted_mistake(name, old, new, pin, tmp_path):
    assert SRC.count(old) == 1, f"mutation site for {name} not found exactly once"
    so = oracle.compile_source(SRC.replace(old, new), str(tmp_path / f"mutant_{name}.so"))
    with oracle.use_library(so):
        with pytest.raises((AssertionError, RuntimeError)):
            pin()
