"""Plant plausible mistakes in copies of the oracle (on the CPU) and check that
the pin battery catches each one: a dropped scale, a flipped sign, a transposed
operand, a wrong index, a dropped term, an unstable grouping, a dropped adapter."""
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

MUTANTS = {
    "dropped_scale": ("d_row[o] += s * acc;", "d_row[o] += acc;"),
    "flipped_sign": ("d_row[o] += s * acc;", "d_row[o] -= s * acc;"),
    "transposed_B": ("acc += widen_bf16(Ba[(int64_t)o * r + j]) * v[j];",
                     "acc += widen_bf16(Ba[(int64_t)j * d_out + o]) * v[j];"),
    "transposed_A": ("acc += widen_bf16(Aa[(int64_t)j * d_in + i]) * widen_bf16(x[i]);",
                     "acc += widen_bf16(Aa[(int64_t)i * r + j]) * widen_bf16(x[i]);"),
    "reversed_x": ("acc += widen_bf16(Aa[(int64_t)j * d_in + i]) * widen_bf16(x[i]);",
                   "acc += widen_bf16(Aa[(int64_t)j * d_in + i]) * widen_bf16(x[d_in - 1 - i]);"),
    "dropped_rank_term": ("        for (int32_t j = 0; j < r; ++j)\n            acc += widen_bf16(Ba",
                          "        for (int32_t j = 0; j + 1 < r; ++j)\n            acc += widen_bf16(Ba"),
    "unstable_route": ("for (int32_t n = 0; n < N; ++n)\n            if (ids[n] == a)",
                       "for (int32_t n = N - 1; n >= 0; --n)\n            if (ids[n] == a)"),
    "merge_transposed_B": ("acc += widen_bf16(Ba[(int64_t)o * r + j]) * widen_bf16(Aa[(int64_t)j * d_in + i]);",
                           "acc += widen_bf16(Ba[(int64_t)j * d_out + o]) * widen_bf16(Aa[(int64_t)j * d_in + i]);"),
    "merge_dropped_base": ("w_row[i] = widen_bf16(W[(int64_t)o * ldw + i]) + scale * acc;",
                           "w_row[i] = scale * acc;"),
    "merge_sign": ("w_row[i] = widen_bf16(W[(int64_t)o * ldw + i]) + scale * acc;",
                   "w_row[i] = widen_bf16(W[(int64_t)o * ldw + i]) - scale * acc;"),
    "linear_wrong_W_column": ("acc += widen_bf16(W[(int64_t)o * ldw + i]) * widen_bf16(x[i]);",
                              "acc += widen_bf16(W[(int64_t)o * ldw + (d_in - 1 - i)]) * widen_bf16(x[i]);"),
    "linear_dropped_base": ("            y_row[o] = acc;\n        }\n        if (seg_ad[sg] == -1)",
                            "            y_row[o] = 0.0 * acc;\n        }\n        if (seg_ad[sg] == -1)"),
    "linear_dropped_delta": ("        if (seg_ad[sg] == -1)\n            continue;\n        int rc = one_adapter(x,",
                             "        if (seg_ad[sg] != -3)\n            continue;\n        int rc = one_adapter(x,"),
    "linear_none_gets_delta": ("        if (seg_ad[sg] == -1)\n            continue;\n        int rc = one_adapter(x,",
                               "        if (seg_ad[sg] == -2)\n            continue;\n        int rc = one_adapter(x,"),
    "dropped_last_adapter": ("for (int32_t p = ad_off[q]; p < ad_off[q + 1]; ++p)",
                             "for (int32_t p = ad_off[q]; p + 1 < ad_off[q + 1]; ++p)"),
}


def _fails(orc):
    failed = []
    for pin in ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, oracle.OracleError):
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(oracle.SOURCE).read()
    assert src.count(old) >= 1, f"mutation site for {name} absent"
    path = os.path.join(tmp_path, f"mut_{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new, 1))  # the first site: the per-token path
    lib = oracle.compile_oracle(path, os.path.join(tmp_path, f"libmut_{name}.so"))
    failed = _fails(oracle.Oracle(lib))
    assert failed, f"mutant {name} passed every pin"
