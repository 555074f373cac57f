"""Pins of the oracle against things other than itself (CPU only).

* store  -> torch ``index_copy_`` (a library routine), bit-exact.
* decode / extend -> dense fp64 SDPA on gathered contiguous K/V (brute force on
  tiny inputs), slot-permutation invariance (bit-identical), closed forms
  (L = 1 gives V; constant V gives that constant; q = 0 or scale = 0 gives the
  mean of V; L = 2 gives the two-key sigmoid form; huge scores give the argmax
  row), causality, and extend/decode consistency.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from mg_testlib import decode_case, dense_decode, dense_extend, extend_case
from paged_kv_attention_mg_b200 import workload as wl

SCALE = 1.0 / math.sqrt(128)


# ----------------------------------------------------------------------------- store

@pytest.mark.parametrize("hkv,seed", [(8, 1), (4, 2), (1, 3)])
def test_store_matches_index_copy(hkv, seed):
    case = extend_case([0, 5, 17], [4, 9, 30], hkv * 2, hkv, seed)
    k_pool = wl.bits(case.k_pool_before).copy()
    v_pool = wl.bits(case.v_pool_before).copy()
    oracle.store_kv(wl.bits(case.data.k_new), wl.bits(case.data.v_new), case.step.out_loc.numpy(),
                    k_pool, v_pool)
    assert np.array_equal(k_pool, wl.bits(case.k_pool))
    assert np.array_equal(v_pool, wl.bits(case.v_pool))
    # slots outside out_loc untouched
    touched = np.zeros(k_pool.shape[0], bool)
    touched[case.step.out_loc.numpy()] = True
    assert np.array_equal(k_pool[~touched], wl.bits(case.k_pool_before)[~touched])


def test_store_rejects_out_of_range_slot():
    case = extend_case([0], [3], 2, 1, 5)
    k_pool = wl.bits(case.k_pool_before).copy()
    v_pool = wl.bits(case.v_pool_before).copy()
    bad = case.step.out_loc.numpy().copy()
    bad[1] = k_pool.shape[0]
    with pytest.raises(oracle.OracleError):
        oracle.store_kv(wl.bits(case.data.k_new), wl.bits(case.data.v_new), bad, k_pool, v_pool)


# ----------------------------------------------------------------------------- decode

DECODE_CASES = [
    # lengths, hq, hkv
    ([5, 9, 12], 16, 8),
    ([1, 2, 3, 40], 8, 8),
    ([33, 7], 8, 2),
    ([17, 1, 64], 16, 2),
    ([25], 32, 4),
    ([3, 31], 4, 1),
    ([11, 4], 12, 4),       # group 3
    ([9, 30], 28, 4),       # group 7
]


@pytest.mark.parametrize("lengths,hq,hkv", DECODE_CASES)
def test_decode_matches_dense_sdpa(lengths, hq, hkv):
    case = decode_case(lengths, hq, hkv, seed=sum(lengths) + hq)
    got = oracle.decode(**case.oracle_args(), scale=SCALE)
    s = case.step
    ref = dense_decode(case.data.q, case.k_pool, case.v_pool, s.page_table, s.table_idx,
                       s.seq_len, SCALE).numpy()
    assert np.isfinite(got).all()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_decode_small_head_dim():
    case = decode_case([6, 11], 4, 2, seed=9, d=16)
    got = oracle.decode(**case.oracle_args(), scale=0.25)
    s = case.step
    ref = dense_decode(case.data.q, case.k_pool, case.v_pool, s.page_table, s.table_idx,
                       s.seq_len, 0.25).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_decode_gqa_mapping_is_consecutive():
    """q heads 2k and 2k+1 share KV head k; another mapping gives other values."""
    case = decode_case([20], 4, 2, seed=4)
    got = oracle.decode(**case.oracle_args(), scale=SCALE)
    s = case.step
    # reference with the modular mapping h -> h % Hkv
    k = case.k_pool[s.page_table[int(s.table_idx[0]), :20].long()].to(torch.float64)
    v = case.v_pool[s.page_table[int(s.table_idx[0]), :20].long()].to(torch.float64)
    q = case.data.q[0].to(torch.float64)
    for h in range(4):
        for kvh, expect_equal in ((h // 2, True), (h % 2, h // 2 == h % 2)):
            x = (k[:, kvh, :] @ q[h]) * SCALE
            w = torch.softmax(x, 0)
            o = (w.unsqueeze(1) * v[:, kvh, :]).sum(0).numpy()
            assert np.allclose(got[0, h], o, atol=1e-12) == expect_equal


def test_decode_slot_permutation_invariance():
    case = decode_case([40, 13, 77], 16, 8, seed=11, num_slots=400)
    args = case.oracle_args()
    base = oracle.decode(**args, scale=SCALE)
    rng = np.random.default_rng(0)
    perm = rng.permutation(args["k_pool"].shape[0])  # slot s moves to perm[s]
    kp = np.empty_like(args["k_pool"]); kp[perm] = args["k_pool"]
    vp = np.empty_like(args["v_pool"]); vp[perm] = args["v_pool"]
    pt = perm[args["page_table"]].astype(np.int32)
    moved = oracle.decode(args["q"], kp, vp, pt, args["table_idx"], args["seq_len"], scale=SCALE)
    assert np.array_equal(base, moved)  # same summation order -> bit-identical


def test_decode_length_one_returns_v():
    case = decode_case([1, 1, 1], 8, 4, seed=3)
    got = oracle.decode(**case.oracle_args(), scale=SCALE)
    s = case.step
    for r in range(3):
        slot = int(s.page_table[int(s.table_idx[r]), 0])
        v = case.v_pool[slot].to(torch.float64).numpy()  # [Hkv, D]
        assert np.array_equal(got[r], np.repeat(v, 2, axis=0))


def test_decode_constant_v_returns_constant():
    case = decode_case([30, 9], 8, 2, seed=5)
    const = torch.randn(2, 128).to(torch.bfloat16)
    for r in range(2):
        slots = case.step.page_table[int(case.step.table_idx[r]), :int(case.step.seq_len[r])].long()
        case.v_pool[slots] = const
    got = oracle.decode(**case.oracle_args(), scale=SCALE)
    want = np.repeat(const.to(torch.float64).numpy(), 4, axis=0)
    for r in range(2):
        np.testing.assert_allclose(got[r], want, rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("zero", ["q", "scale"])
def test_decode_uniform_weights_give_mean(zero):
    case = decode_case([13, 50], 8, 4, seed=6)
    args = case.oracle_args()
    scale = SCALE
    if zero == "q":
        args["q"] = np.zeros_like(args["q"])
    else:
        scale = 0.0
    got = oracle.decode(**args, scale=scale)
    s = case.step
    for r in range(2):
        L = int(s.seq_len[r])
        slots = s.page_table[int(s.table_idx[r]), :L].long()
        mean = case.v_pool[slots].to(torch.float64).mean(0).numpy()
        np.testing.assert_allclose(got[r], np.repeat(mean, 2, axis=0), rtol=0, atol=1e-13)


def test_decode_two_keys_sigmoid_form():
    case = decode_case([2, 2], 4, 2, seed=8)
    got = oracle.decode(**case.oracle_args(), scale=SCALE)
    s = case.step
    for r in range(2):
        slots = s.page_table[int(s.table_idx[r]), :2].long()
        k = case.k_pool[slots].to(torch.float64).numpy()
        v = case.v_pool[slots].to(torch.float64).numpy()
        q = case.data.q[r].to(torch.float64).numpy()
        for h in range(4):
            kvh = h // 2
            x0 = SCALE * float(q[h] @ k[0, kvh])
            x1 = SCALE * float(q[h] @ k[1, kvh])
            s0 = 1.0 / (1.0 + math.exp(x1 - x0))
            s1 = 1.0 / (1.0 + math.exp(x0 - x1))
            np.testing.assert_allclose(got[r, h], s0 * v[0, kvh] + s1 * v[1, kvh], atol=1e-13)


def test_decode_huge_scores_pick_argmax_row():
    """With a very large scale softmax is one-hot: needs the max subtraction."""
    case = decode_case([21], 2, 1, seed=12)
    got = oracle.decode(**case.oracle_args(), scale=1e4)
    s = case.step
    slots = s.page_table[int(s.table_idx[0]), :21].long()
    k = case.k_pool[slots].to(torch.float64)[:, 0, :]
    v = case.v_pool[slots].to(torch.float64)[:, 0, :]
    for h in range(2):
        j = int(torch.argmax(k @ case.data.q[0, h].to(torch.float64)))
        np.testing.assert_allclose(got[0, h], v[j].numpy(), atol=1e-12)


def test_decode_request_subset_leaves_others_untouched():
    case = decode_case([7, 8, 9], 4, 2, seed=13)
    full = oracle.decode(**case.oracle_args(), scale=SCALE)
    part = oracle.decode(**case.oracle_args(), scale=SCALE, requests=[1])
    assert np.array_equal(part[1], full[1])
    assert np.isnan(part[0]).all() and np.isnan(part[2]).all()


def test_decode_threads_do_not_change_bits():
    case = decode_case([100, 37, 5, 64], 16, 4, seed=14)
    a = oracle.decode(**case.oracle_args(), scale=SCALE, threads=1)
    b = oracle.decode(**case.oracle_args(), scale=SCALE, threads=4)
    assert np.array_equal(a, b)


def test_decode_rejects_bad_metadata():
    case = decode_case([5, 6], 4, 2, seed=15)
    args = case.oracle_args()
    bad = dict(args, seq_len=np.array([5, args["page_table"].shape[1] + 1], np.int32))
    with pytest.raises(oracle.OracleError):
        oracle.decode(**bad, scale=SCALE)
    bad = dict(args, table_idx=np.array([0, 99], np.int32))
    with pytest.raises(oracle.OracleError):
        oracle.decode(**bad, scale=SCALE)
    pt = args["page_table"].copy()
    pt[int(args["table_idx"][0]), 0] = -5
    with pytest.raises(oracle.OracleError):
        oracle.decode(**dict(args, page_table=pt), scale=SCALE)


# ----------------------------------------------------------------------------- extend

EXTEND_CASES = [
    # cached, seq, hq, hkv
    ([0, 3, 10], [4, 9, 11], 16, 8),
    ([0], [37], 8, 2),
    ([20, 0, 5], [21, 33, 70], 8, 1),
    ([64, 1], [90, 3], 32, 4),
    ([3, 0], [10, 40], 12, 4),      # group 3
]


def _extend_args(case):
    s = case.step
    a = case.oracle_args()
    a.update(cached_len=s.cached_len.numpy(), q_offset=s.q_offset.numpy())
    return a


@pytest.mark.parametrize("cached,seq,hq,hkv", EXTEND_CASES)
def test_extend_matches_dense_causal_sdpa(cached, seq, hq, hkv):
    case = extend_case(cached, seq, hq, hkv, seed=sum(seq) + 7 * hq)
    got = oracle.extend(**_extend_args(case), scale=SCALE)
    s = case.step
    ref = dense_extend(case.data.q, case.k_pool, case.v_pool, s.page_table, s.table_idx,
                       s.cached_len, s.seq_len, s.q_offset, SCALE).numpy()
    assert np.isfinite(got).all()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_extend_single_new_token_equals_decode():
    case = extend_case([4, 8, 11], [5, 9, 12], 16, 8, seed=21)
    ext = oracle.extend(**_extend_args(case), scale=SCALE)
    dec = oracle.decode(**case.oracle_args(), scale=SCALE)
    assert np.array_equal(ext, dec)


def test_extend_rows_equal_truncated_decodes():
    """Row i of request r equals a decode whose context ends at position c+i."""
    case = extend_case([6, 0], [15, 7], 8, 4, seed=22)
    args = _extend_args(case)
    ext = oracle.extend(**args, scale=SCALE)
    s = case.step
    for r in range(2):
        c, L = int(s.cached_len[r]), int(s.seq_len[r])
        for i in range(L - c):
            t = int(s.q_offset[r]) + i
            dec = oracle.decode(args["q"][t:t + 1].copy(), args["k_pool"], args["v_pool"],
                                args["page_table"], args["table_idx"][r:r + 1].copy(),
                                np.array([c + i + 1], np.int32), scale=SCALE)
            assert np.array_equal(ext[t], dec[0])


def test_extend_is_causal():
    """Changing K/V at positions after c+i does not change row i."""
    case = extend_case([3], [12], 4, 2, seed=23)
    args = _extend_args(case)
    base = oracle.extend(**args, scale=SCALE)
    s = case.step
    row = s.page_table[int(s.table_idx[0])]
    kp, vp = args["k_pool"].copy(), args["v_pool"].copy()
    late = row[3 + 5 + 1:12].numpy()  # positions after c + 5
    kp[late] = wl.bits(torch.randn(len(late), 2, 128).to(torch.bfloat16))
    vp[late] = wl.bits(torch.randn(len(late), 2, 128).to(torch.bfloat16))
    moved = oracle.extend(**dict(args, k_pool=kp, v_pool=vp), scale=SCALE)
    assert np.array_equal(base[:6], moved[:6])
    assert not np.allclose(base[6:], moved[6:])


def test_extend_slot_permutation_invariance():
    case = extend_case([10, 0, 31], [40, 25, 35], 8, 2, seed=24, num_slots=300)
    args = _extend_args(case)
    base = oracle.extend(**args, scale=SCALE)
    perm = np.random.default_rng(1).permutation(args["k_pool"].shape[0])
    kp = np.empty_like(args["k_pool"]); kp[perm] = args["k_pool"]
    vp = np.empty_like(args["v_pool"]); vp[perm] = args["v_pool"]
    pt = perm[args["page_table"]].astype(np.int32)
    moved = oracle.extend(**dict(args, k_pool=kp, v_pool=vp, page_table=pt), scale=SCALE)
    assert np.array_equal(base, moved)


def test_extend_zero_new_tokens_is_empty():
    case = extend_case([5, 7], [5, 9], 4, 2, seed=25)
    got = oracle.extend(**_extend_args(case), scale=SCALE)
    assert got.shape[0] == 2 and np.isfinite(got).all()


def test_extend_rejects_inconsistent_offsets():
    case = extend_case([1, 2], [4, 6], 4, 2, seed=26)
    args = _extend_args(case)
    bad = args["q_offset"].copy()
    bad[1] += 1
    with pytest.raises(oracle.OracleError):
        oracle.extend(**dict(args, q_offset=bad), scale=SCALE)
