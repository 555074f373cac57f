"""Planted mistakes: each plausible bug, planted in a copy of the oracle's C
source on the CPU, must make at least one pin fail.  This shows the pins can
tell a right oracle from a wrong one (a dropped term, a wrong index, a
transposed operand, an off-by-one mask)."""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from mg_testlib import decode_case, dense_decode, dense_extend, extend_case
from paged_kv_attention_mg_b200 import workload as wl

SCALE = 1.0 / math.sqrt(128)

MUTANTS = {
    "gqa_modular_mapping": ("L - 1, h / group,", "L - 1, h % num_kv_heads,"),
    "dropped_scale": ("x[j] = scale * dot;", "x[j] = dot;"),
    "dropped_max_subtraction": ("double w = exp(x[j] - x_max);", "double w = exp(x[j]);"),
    "v_read_from_k_pool": ("const uint16_t *v_vec = v_pool +", "const uint16_t *v_vec = k_pool +"),
    "no_normalisation": ("o[d] /= denom;", "o[d] /= 1.0;"),
    "decode_skips_new_token": ("L - 1, h / group,", "L - 2 < 0 ? 0 : L - 2, h / group,"),
    "extend_mask_excludes_diagonal": ("pt_row, c + i, h / group,", "pt_row, c + i - 1 < 0 ? 0 : c + i - 1, h / group,"),
    "extend_mask_one_key_late": ("pt_row, c + i, h / group,", "pt_row, c + i + 1 < c + n ? c + i + 1 : c + i, h / group,"),
    "extend_wrong_query_row": ("const int64_t t = q_offset[r] + i;", "const int64_t t = q_offset[r];"),
    "store_swaps_k_and_v": ("= k[t * row + h * head_dim + d];", "= v[t * row + h * head_dim + d];"),
    "dot_uses_wrong_dim_of_q": ("bf16_bits_to_double(q_vec[d]) *", "bf16_bits_to_double(q_vec[0]) *"),
    "decode_row_ignores_table_idx": ("num_slots, page_table + (int64_t)table_idx[r] * pt_stride,",
                                     "num_slots, page_table + (int64_t)r * pt_stride,"),
    "extend_row_ignores_table_idx": ("*pt_row = page_table + (int64_t)table_idx[r] * pt_stride;",
                                     "*pt_row = page_table + (int64_t)r * pt_stride;"),
    "extend_attends_only_to_the_chunk": ("pt_row, c + i, h / group,", "pt_row + c, i, h / group,"),
    "v_row_of_the_previous_key": ("v_pool + (int64_t)pt_row[j] * row", "v_pool + (int64_t)pt_row[j > 0 ? j - 1 : 0] * row"),
    "decode_length_of_the_table_row": ("const int64_t L = seq_len[r];", "const int64_t L = seq_len[table_idx[r]];"),
    "store_tokens_in_reverse": ("int64_t slot = out_loc[t];", "int64_t slot = out_loc[num_tokens - 1 - t];"),
    "v_from_kv_head_zero": ("row + kvh * head_dim;\n        for (int64_t d = 0; d < head_dim; ++d) o[d] +=",
                            "row + 0 * head_dim;\n        for (int64_t d = 0; d < head_dim; ++d) o[d] +="),
}


def _pins(lib):
    """A compact battery of the pins in test_oracle_pins.py; returns failures."""
    failures = []
    # store vs index_copy
    case = extend_case([0, 5], [4, 9], 8, 4, seed=101)
    kp = wl.bits(case.k_pool_before).copy()
    vp = wl.bits(case.v_pool_before).copy()
    try:
        oracle.store_kv(wl.bits(case.data.k_new), wl.bits(case.data.v_new),
                        case.step.out_loc.numpy(), kp, vp, lib=lib)
        if not (np.array_equal(kp, wl.bits(case.k_pool)) and np.array_equal(vp, wl.bits(case.v_pool))):
            failures.append("store")
    except oracle.OracleError:
        failures.append("store-error")
    # decode vs dense SDPA
    case = decode_case([5, 9, 12, 2], 16, 4, seed=104)
    s = case.step
    # no request reads page-table row r itself, so a mix-up of r and table_idx[r] shows
    assert all(int(t) != r for r, t in enumerate(s.table_idx.tolist()))
    try:
        got = oracle.decode(**case.oracle_args(), scale=SCALE, lib=lib)
        ref = dense_decode(case.data.q, case.k_pool, case.v_pool, s.page_table, s.table_idx,
                           s.seq_len, SCALE).numpy()
        if not np.allclose(got, ref, rtol=0, atol=1e-12):
            failures.append("decode-dense")
    except oracle.OracleError:
        failures.append("decode-error")
    # huge scores -> argmax row
    case = decode_case([21], 2, 1, seed=12)
    s = case.step
    try:
        got = oracle.decode(**case.oracle_args(), scale=1e4, lib=lib)
        slots = s.page_table[int(s.table_idx[0]), :21].long()
        k = case.k_pool[slots].to(torch.float64)[:, 0, :]
        v = case.v_pool[slots].to(torch.float64)[:, 0, :]
        j = int(torch.argmax(k @ case.data.q[0, 0].to(torch.float64)))
        if not np.allclose(got[0, 0], v[j].numpy(), atol=1e-12):
            failures.append("argmax")
    except oracle.OracleError:
        failures.append("argmax-error")
    # extend vs dense causal SDPA
    case = extend_case([0, 3, 10], [4, 9, 14], 8, 2, seed=103)
    s = case.step
    assert all(int(t) != r for r, t in enumerate(s.table_idx.tolist()))
    try:
        a = case.oracle_args()
        a.update(cached_len=s.cached_len.numpy(), q_offset=s.q_offset.numpy())
        got = oracle.extend(**a, scale=SCALE, lib=lib)
        ref = dense_extend(case.data.q, case.k_pool, case.v_pool, s.page_table, s.table_idx,
                           s.cached_len, s.seq_len, s.q_offset, SCALE).numpy()
        if not np.allclose(got, ref, rtol=0, atol=1e-12):
            failures.append("extend-dense")
    except oracle.OracleError:
        failures.append("extend-error")
    return failures


def test_unmutated_oracle_passes_battery():
    assert _pins(oracle.load()) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    before, after = MUTANTS[name]
    src = open(oracle.SOURCE).read()
    assert src.count(before) == 1, f"mutation anchor for {name} not unique/found"
    path = os.path.join(tmp_path, f"mutant_{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(before, after))
    lib = oracle.load(oracle.build(path, os.path.join(tmp_path, f"lib{name}.so"), force=True))
    assert _pins(lib), f"planted mistake {name} was not caught by any pin"
