"""Pins for the CPU oracle: each test ties the oracle to something other than itself --
a worked example printed on the pages (tests/golden/, with citations), a closed form,
an invariant, an independent formulation (pad/even-exchange/trim, stable sort), a
library routine (torch's bf16 / float8_e4m3fn casts) or pure-Python brute force on tiny
inputs -- chosen so that a dropped term, a wrong sign or index or a transposed operand
anywhere in the oracle fails at least one of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


# ------------------------------------------------------------------ helpers

def brute_all_to_all(S, sends):
    """Pure-Python exchange: rank j's send list is cut, in destination order, into chunks
    of S[j][0], S[j][1], ...; rank i receives chunk i of every rank, in rank order."""
    W = len(S)
    recv = [[] for _ in range(W)]
    for j in range(W):
        pos = 0
        for i in range(W):
            recv[i].extend(sends[j][pos:pos + S[j][i]])
            pos += S[j][i]
    return recv


def pad_even_trim(S, sends, cap):
    """Second formulation of an uneven all-to-all (torch-neuronx PR, Motivation and
    Context): every sender pads each of its chunks to `cap` rows, one even all-to-all
    swaps equal-sized blocks, every receiver trims each block to the size it expects."""
    W = len(S)
    padded = []
    for j in range(W):
        pos, blocks = 0, []
        for i in range(W):
            chunk = list(sends[j][pos:pos + S[j][i]])
            pos += S[j][i]
            blocks.append(chunk + [None] * (cap - len(chunk)))
        padded.append(blocks)
    even = [[padded[j][i] for j in range(W)] for i in range(W)]     # even all-to-all
    out_splits = [[S[j][i] for j in range(W)] for i in range(W)]    # receiver's view
    return [[row for j in range(W) for row in even[i][j][:out_splits[i][j]]]
            for i in range(W)]


def run_oracle_a2a(S, rows_per_rank, cols, label=lambda i, k: 10 * i + k, plan=None):
    W = len(S)
    inp = np.zeros((W, rows_per_rank, cols), np.float32)
    for i in range(W):
        for k in range(rows_per_rank):
            inp[i, k, :] = label(i, k)
    src, out_s, dst, fl = oracle.a2a_exchange_plan(np.array(S))
    assert fl == 0
    if plan is not None:
        src, out_s, dst = plan(src, out_s, dst)
    cap_out = max(1, int(np.asarray(S).sum(axis=0).max()))
    out = np.full((W, cap_out, cols), -1.0, np.float32)
    fl = oracle.a2a_v(inp, out, src, out_s, dst)
    n = out_s.sum(axis=1)
    return out, n, fl


# ------------------------------------------------------------ O1 / O2 pins

def test_p3_worked_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "p3_uneven_a2a_2rank.json")))
    out, n, fl = run_oracle_a2a(g["in_splits"], g["rows_per_rank"], g["cols"])
    assert fl == 0
    for i, exp in enumerate(g["expected_rows"]):
        assert int(n[i]) == len(exp)
        got = out[i, :len(exp)]
        assert (got == np.array(exp, np.float32)[:, None]).all(), (i, got[:, 0])
        assert (out[i, len(exp):] == -1).all()          # rows past the receive count untouched


@pytest.mark.parametrize("bug", ["rows_from_block_start", "splits_swapped"])
def test_old_lowering_bugs_are_caught(golden_dir, bug):
    """The two data bugs the torch-neuronx PR lists for the old lowering (rows for rank r
    taken from the start of each sender's block; input and output split operands
    swapped), planted in the oracle's plan here on the CPU, must fail the worked example."""
    g = json.load(open(os.path.join(golden_dir, "p3_uneven_a2a_2rank.json")))
    if bug == "rows_from_block_start":
        plan = lambda s, o, d: (np.zeros_like(s), o, d)
    else:
        plan = lambda s, o, d: (s, o.T.copy(), np.concatenate(
            [np.zeros((o.shape[0], 1), np.int64), np.cumsum(o.T, axis=1)[:, :-1]], axis=1))
    out, n, fl = run_oracle_a2a(g["in_splits"], g["rows_per_rank"], g["cols"], plan=plan)
    ok = all(int(n[i]) == len(e) and (out[i, :len(e), 0] == np.array(e)).all()
             for i, e in enumerate(g["expected_rows"]))
    assert not ok


def test_two_dimensional_rows_and_one_column(golden_dir):
    """The first old-lowering bug was 1-D-only types: the oracle must move [rows, cols]
    rows of any width, including 1 column."""
    g = json.load(open(os.path.join(golden_dir, "p3_uneven_a2a_2rank.json")))
    for cols in (1, 8, 33):
        out, n, fl = run_oracle_a2a(g["in_splits"], g["rows_per_rank"], cols)
        for i, exp in enumerate(g["expected_rows"]):
            assert (out[i, :len(exp)] == np.array(exp, np.float32)[:, None]).all()


def test_plan_matches_p1_test_semantics():
    """test_make_a2a_exchange_plan: out_splits is the all_to_all_single of in_splits,
    src_offsets the all_to_all_single of the exclusive scan of in_splits, dst_offsets[0]
    is 0 and dst_offsets[1:] the inclusive scan of out_splits without its last entry;
    in_splits is unchanged. all_to_all_single is simulated chunk by chunk here."""
    rng = np.random.default_rng(7)
    for W in (1, 2, 3, 5, 8, 17):
        S = rng.integers(0, 10, size=(W, W))
        S0 = S.copy()
        src, out, dst, fl = oracle.a2a_exchange_plan(S)
        assert fl == 0 and (S == S0).all()
        excl = [[sum(S[j][:i]) for i in range(W)] for j in range(W)]   # per rank j
        for i in range(W):
            for j in range(W):
                assert out[i][j] == S[j][i]            # chunk i of rank j's in_splits
                assert src[i][j] == excl[j][i]         # chunk i of rank j's scan
            assert dst[i][0] == 0
            assert list(dst[i][1:]) == list(np.cumsum(out[i])[:-1])


@pytest.mark.parametrize("seed", range(12))
def test_a2a_matches_brute_force_and_pad_trim(seed):
    rng = np.random.default_rng(seed)
    W = int(rng.integers(1, 7))
    S = rng.integers(0, 5, size=(W, W))
    S[rng.random((W, W)) < 0.3] = 0                     # zero-row chunks
    rows = max(1, int(S.sum(axis=1).max()))
    label = lambda i, k: 1000 * i + k
    out, n, fl = run_oracle_a2a(S.tolist(), rows, 3, label=label)
    assert fl == 0
    sends = [[label(j, k) for k in range(rows)] for j in range(W)]
    bf = brute_all_to_all(S.tolist(), sends)
    pt = pad_even_trim(S.tolist(), sends, max(1, int(S.max())))
    assert bf == pt
    for i in range(W):
        assert int(n[i]) == len(bf[i])
        assert out[i, :len(bf[i]), 0].tolist() == bf[i]


def test_a2a_rejects_out_of_range_segments():
    S = np.array([[2, 1], [1, 2]])
    src, out_s, dst, _ = oracle.a2a_exchange_plan(S)
    inp = np.arange(2 * 3 * 4, dtype=np.float32).reshape(2, 3, 4)
    out = np.full((2, 2, 4), -7, np.float32)           # capacity 2 < 3 received rows
    fl = oracle.a2a_v(inp, out, src, out_s, dst)
    assert fl & oracle.ORC_BAD_SPLIT
    neg = np.array([[1, -1], [0, 0]])
    assert oracle.a2a_exchange_plan(neg)[3] & oracle.ORC_BAD_SPLIT


# --------------------------------------------------------------- O3 pins

def brute_layout(W, T, K, E, ids, active):
    """The 2-D expert-major layout by definition, in nested loops: destination rank d's
    receive buffer holds, for each of its local experts le in order, for each source
    rank r in order, r's slots that chose expert d*ne+le, in slot order."""
    ne = E // W
    rows = []
    for d in range(W):
        for le in range(ne):
            e = d * ne + le
            for r in range(W):
                for t in range(T):
                    g = r * T + t
                    for k in range(K):
                        if active is not None:
                            flag = active[g][k] if isinstance(active[g], (list, tuple)) else active[g]
                            if not flag:
                                continue
                        if ids[g][k] == e:
                            rows.append(g * K + k)
    dst_row = [-1] * (W * T * K)
    for pos, s in enumerate(rows):
        dst_row[s] = pos
    return rows, dst_row


def test_p1_occurrence_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "p1_occurrence_numbers.json")))
    vals = g["values"]
    lay = oracle.moe_dispatch_layout(1, len(vals), 1, 4, np.array(vals, np.int32))
    assert lay["occ"].tolist() == g["expected_occurrence"]
    assert lay["occ"].tolist() != g["docstring_one_based"]


def _check_layout(W, T, K, E, ids, active, lay):
    G = W * T
    ne = E // W
    ids2 = np.asarray(ids).reshape(G, K)
    if active is None:
        act = np.ones(G * K, bool)
    else:
        a = np.asarray(active).astype(bool)
        act = np.repeat(a.reshape(-1), K) if a.ndim == 1 else a.reshape(-1)
    slot_active = act & (ids2.reshape(-1) >= 0) & (ids2.reshape(-1) < E)
    R = int(slot_active.sum())
    assert lay["R"] == R
    # closed form: dst_row = position in a stable sort of the active slots by expert id
    s_act = np.nonzero(slot_active)[0]
    order = s_act[np.argsort(ids2.reshape(-1)[s_act], kind="stable")]
    exp = np.full(G * K, -1, np.int64)
    exp[order] = np.arange(R)
    assert (lay["dst_row"] == exp).all()
    # bijection and inverse
    assert sorted(lay["dst_row"][slot_active].tolist()) == list(range(R))
    assert (lay["assist_info"][lay["dst_row"][slot_active]] == np.nonzero(slot_active)[0]).all()
    # counts
    cnt = np.zeros((W, E), np.int64)
    for s in s_act:
        cnt[(s // K) // T, ids2.reshape(-1)[s]] += 1
    assert (lay["cnt"] == cnt).all()
    assert (lay["cnt"].sum(axis=1) == slot_active.reshape(W, T * K).sum(axis=1)).all()
    # expert_base / rank_base / send_splits
    tot = cnt.sum(axis=0)
    assert lay["expert_base"].tolist() == [0] + np.cumsum(tot).tolist()
    assert lay["rank_base"].tolist() == [int(lay["expert_base"][d * ne]) for d in range(W)] + [R]
    assert (lay["send_splits"] == cnt.reshape(W, W, ne).sum(axis=2)).all()
    # occ: 0-based count of earlier active slots of the same source rank and expert
    seen = {}
    for s in range(G * K):
        if not slot_active[s]:
            assert lay["occ"][s] == -1 and lay["dst_row"][s] == -1
            continue
        key = ((s // K) // T, int(ids2.reshape(-1)[s]))
        assert lay["occ"][s] == seen.get(key, 0)
        seen[key] = seen.get(key, 0) + 1


@pytest.mark.parametrize("seed", range(10))
def test_layout_brute_force_tiny(seed):
    rng = np.random.default_rng(100 + seed)
    W = int(rng.integers(1, 5))
    ne = int(rng.integers(1, 4))
    E = W * ne
    T = int(rng.integers(0, 7))
    K = int(rng.integers(1, 4))
    ids = rng.integers(0, E, size=(W * T, K)).astype(np.int32)      # duplicates allowed
    active = (rng.random(W * T) < 0.7).astype(np.uint8) if seed % 2 else None
    lay = oracle.moe_dispatch_layout(W, T, K, E, ids, active)
    assert lay["flags"] == 0
    rows, dst_row = brute_layout(W, T, K, E, ids.tolist(),
                                 None if active is None else active.tolist())
    assert lay["dst_row"].tolist() == dst_row
    assert lay["assist_info"][:len(rows)].tolist() == rows
    _check_layout(W, T, K, E, ids, active, lay)


@pytest.mark.parametrize("seed", range(6))
def test_layout_slot_mask_brute_force_tiny(seed):
    """[P4] 2-D xActiveMask (Bs, K): each slot's own flag decides; nested-loop brute force."""
    rng = np.random.default_rng(200 + seed)
    W = int(rng.integers(1, 5))
    ne = int(rng.integers(1, 4))
    E = W * ne
    T = int(rng.integers(1, 7))
    K = int(rng.integers(2, 5))
    ids = rng.integers(0, E, size=(W * T, K)).astype(np.int32)
    active = (rng.random((W * T, K)) < 0.6).astype(np.uint8)
    active[0] = 0                                                  # a token that sends nothing
    lay = oracle.moe_dispatch_layout(W, T, K, E, ids, active)
    assert lay["flags"] == 0
    rows, dst_row = brute_layout(W, T, K, E, ids.tolist(), active.tolist())
    assert lay["dst_row"].tolist() == dst_row
    assert lay["assist_info"][:len(rows)].tolist() == rows
    assert (lay["dst_row"][:K] == -1).all() and (lay["occ"][:K] == -1).all()
    _check_layout(W, T, K, E, ids, active, lay)


def test_layout_slot_mask_repeating_token_mask_equals_token_mask():
    w = wl.moe_workload("tiny", seed=21, W=3, T=40, E=12, K=3, active_p=0.6)
    one = oracle.moe_dispatch_layout(w.W, w.T, w.K, w.E, w.expert_ids, w.active)
    two = oracle.moe_dispatch_layout(w.W, w.T, w.K, w.E, w.expert_ids,
                                     np.repeat(w.active[:, None], w.K, axis=1))
    for k in ("cnt", "occ", "dst_row", "expert_base", "rank_base", "send_splits"):
        assert np.array_equal(one[k], two[k]), k
    assert np.array_equal(one["assist_info"][:one["R"]], two["assist_info"][:two["R"]])


@pytest.mark.parametrize("name,over", [("tiny", {}), ("tiny", dict(W=3, T=37, E=12, K=3)),
                                       ("tiny", dict(W=4, T=50, E=16, K=4, slot_active_p=0.5)),
                                       ("cfg4", dict(T=64)), ("cfg3", dict(T=128, H=256))])
def test_layout_closed_form_on_workloads(name, over):
    w = wl.moe_workload(name, seed=3, **over)
    lay = oracle.moe_dispatch_layout(w.W, w.T, w.K, w.E, w.expert_ids, w.active)
    assert lay["flags"] == 0
    _check_layout(w.W, w.T, w.K, w.E, w.expert_ids, w.active, lay)


@pytest.mark.parametrize("A", [2, 3, 8, 128])
@pytest.mark.parametrize("seed", range(3))
def test_layout_major_align_properties(A, seed):
    """[P1] all_to_all_vdev_2d major_align: every expert segment starts on a multiple of A,
    holds the expert's rows in stable slot order and then padding rows (assist_info -1),
    is a multiple of A long, never empty, and pads by less than A past its rows; every
    dst_row moves by its expert's base shift only."""
    rng = np.random.default_rng(300 + seed)
    W, ne = int(rng.integers(1, 5)), int(rng.integers(1, 5))
    E, T, K = W * ne, int(rng.integers(1, 40)), int(rng.integers(1, 4))
    ids = rng.integers(0, E, size=(W * T, K)).astype(np.int32)
    ids[ids == E - 1] = 0                                          # expert E-1 stays empty
    active = (rng.random(W * T) < 0.8).astype(np.uint8)
    plain = oracle.moe_dispatch_layout(W, T, K, E, ids, active)
    pad = oracle.moe_dispatch_layout(W, T, K, E, ids, active, major_align=A)
    assert pad["flags"] == 0
    eb, eb0 = pad["expert_base"], plain["expert_base"]
    rows, _ = brute_layout(W, T, K, E, ids.tolist(), active.tolist())
    pos = 0
    for e in range(E):
        n = int(eb0[e + 1] - eb0[e])
        seg = int(eb[e + 1] - eb[e])
        assert eb[e] % A == 0 and seg % A == 0 and seg >= n
        assert seg == A if n == 0 else seg - n < A
        assert pad["assist_info"][eb[e]:eb[e] + n].tolist() == rows[pos:pos + n]
        assert (pad["assist_info"][eb[e] + n:eb[e + 1]] == -1).all()
        pos += n
    assert eb[E - 1 + 1] - eb[E - 1] == A                          # the empty expert
    act = plain["dst_row"] >= 0
    e_of = ids.reshape(-1)
    assert (pad["dst_row"][~act] == -1).all()
    assert (pad["dst_row"][act] - plain["dst_row"][act] == (eb - eb0)[e_of[act]]).all()
    assert pad["rank_base"].tolist() == [int(eb[d * ne]) for d in range(W)] + [int(eb[E])]
    for k in ("cnt", "occ", "send_splits"):
        assert np.array_equal(pad[k], plain[k]), k


def test_layout_major_align_one_is_no_padding():
    w = wl.moe_workload("tiny", seed=22, W=3, T=30, E=12, K=3, active_p=0.7)
    base = oracle.moe_dispatch_layout(w.W, w.T, w.K, w.E, w.expert_ids, w.active)
    for A in (0, 1):
        o = oracle.moe_dispatch_layout(w.W, w.T, w.K, w.E, w.expert_ids, w.active, major_align=A)
        for k in ("cnt", "occ", "dst_row", "expert_base", "rank_base", "send_splits"):
            assert np.array_equal(o[k], base[k]), k


def test_recv_counts_major_align_absorbed_by_last_rank():
    """As in [P1]'s 2-D plan test, the last source rank's split absorbs the padding:
    per expert the received counts sum to the padded segment."""
    w = wl.moe_workload("tiny", seed=23, W=4, T=9, E=12, K=3)
    A = 8
    lay = oracle.moe_dispatch_layout(w.W, w.T, w.K, w.E, w.expert_ids, w.active, major_align=A)
    ne = w.E // w.W
    etn1, erc, _ = oracle.moe_recv_counts(w.W, w.E, lay["cnt"], 1, major_align=A)
    etn0, _, _ = oracle.moe_recv_counts(w.W, w.E, lay["cnt"], 0, major_align=A)
    seg = np.diff(lay["expert_base"]).reshape(w.W, ne)
    assert (erc.sum(axis=2) == seg).all() and (etn1 == seg).all()
    assert (erc[:, :, :-1] == lay["cnt"].T.reshape(w.W, ne, w.W)[:, :, :-1]).all()
    assert (etn0[:, -1] == np.diff(lay["rank_base"])).all()


def test_layout_bad_expert_and_capacity():
    ids = np.array([[0, 5], [1, -1], [2, 3]], np.int32)     # W=1, T=3, K=2, E=4
    lay = oracle.moe_dispatch_layout(1, 3, 2, 4, ids)
    assert lay["flags"] & oracle.ORC_BAD_EXPERT
    assert lay["dst_row"].tolist() == [0, -1, 1, -1, 2, 3]
    lay = oracle.moe_dispatch_layout(1, 3, 2, 4, np.array([[0, 1], [1, 2], [2, 3]], np.int32),
                                     rows_cap=4)
    assert lay["flags"] & oracle.ORC_CAPACITY
    assert (lay["assist_info"][:4] >= 0).all()


def test_recv_counts_against_dispatched_rows():
    """ep_recv_counts and expert_token_nums re-derived from where the rows actually
    landed (assist_info -> slot -> source rank), not from cnt."""
    w = wl.moe_workload("tiny", seed=5, W=4, T=9, E=12, K=3)
    ne = w.E // w.W
    lay = oracle.moe_dispatch_layout(w.W, w.T, w.K, w.E, w.expert_ids, w.active)
    etn1, erc, _ = oracle.moe_recv_counts(w.W, w.E, lay["cnt"], 1)
    etn0, _, _ = oracle.moe_recv_counts(w.W, w.E, lay["cnt"], 0)
    ids = w.expert_ids.reshape(-1)
    exp_rc = np.zeros((w.W, ne, w.W), np.int64)
    for row in range(lay["R"]):
        s = lay["assist_info"][row]
        e = ids[s]
        exp_rc[e // ne, e % ne, (s // w.K) // w.T] += 1
        d = e // ne
        assert lay["rank_base"][d] <= row < lay["rank_base"][d + 1]
    assert (erc == exp_rc).all()
    assert (etn1 == exp_rc.sum(axis=2)).all()
    assert (etn0 == np.cumsum(exp_rc.sum(axis=2), axis=1)).all()
    assert (etn0[:, -1] == np.diff(lay["rank_base"])).all()


# --------------------------------------------------------------- O4 pins

def test_bf16_conversion_matches_torch():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 20000),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, 1e-40], np.float32)])
    v = v.astype(np.float32)
    # ties: values exactly halfway between two bf16 numbers
    base = wl.bf16_bits_to_f32(rng.integers(0, 0x7f00, 2000).astype(np.uint16))
    ties = (base.view(np.uint32) | 0x8000).view(np.float32)
    v = np.concatenate([v, ties, -ties]).astype(np.float32)
    exp = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_from_f32(float(x)) for x in v], np.uint16)
    assert (got == exp).all()


def test_e4m3_decode_all_codes_matches_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).float().numpy()
    got = np.array([oracle.e4m3_to_f32(c) for c in range(256)], np.float32)
    nan = np.isnan(ref)
    assert (np.isnan(got) == nan).all() and nan.sum() == 2          # S.1111.111
    assert (got[~nan] == ref[~nan]).all()
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def test_e4m3_encode_matches_torch_in_range_and_saturates():
    rng = np.random.default_rng(1)
    grid = np.array([oracle.e4m3_to_f32(c) for c in range(0x7F)], np.float64)  # >= 0
    mids = (grid[:-1] + grid[1:]) / 2
    v = np.concatenate([grid, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
                        rng.uniform(-464, 464, 30000), rng.standard_normal(5000) * 1e-3])
    v = np.concatenate([v, -v]).astype(np.float32)
    v = v[np.abs(v) <= 464]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_from_f32(float(x)) for x in v], np.uint8)
    # torch maps -0 and +0 to their own codes as well
    assert (got == ref).all(), v[got != ref][:10]
    for big in (464.0001, 479.0, 480.0, 1e6):                  # satfinite: +-448, not NaN
        assert oracle.e4m3_from_f32(big) == 0x7E
        assert oracle.e4m3_from_f32(-big) == 0xFE


def _quant_brute(xf, mode):
    """Quantisation with a different arithmetic path: fp32 quotients via double division
    of fp32 operands (correctly rounded to fp32, since 53 >= 2*24+2), Python's
    round-half-even, and for e4m3 torch's cast."""
    qmax = 127.0 if mode == 2 else 448.0
    amax = max(abs(float(a)) for a in xf)
    scale = float(np.float32(amax / qmax))
    if amax == 0:
        return [0] * len(xf), 0.0
    vals = [float(np.float32(float(a) / scale)) for a in xf]
    if mode == 2:
        return [max(-127, min(127, round(v))) & 0xFF for v in vals], scale
    ref = torch.tensor(vals, dtype=torch.float32).clamp(-448, 448).to(torch.float8_e4m3fn)
    return ref.view(torch.uint8).tolist(), scale


@pytest.mark.parametrize("mode", [2, 3])
def test_quant_row_brute_force(mode):
    w = wl.moe_workload("tiny", seed=11, T=8, H=64, outlier_frac=0.1, zero_rows=0.05)
    for g in range(w.G):
        q, s = oracle.quant_row(w.x_bits[g], mode)
        xf = wl.bf16_bits_to_f32(w.x_bits[g])
        qb, sb = _quant_brute(xf, mode)
        assert s == np.float32(sb)
        assert q.tolist() == qb


@pytest.mark.parametrize("mode", [2, 3])
def test_quant_properties(mode):
    w = wl.moe_workload("cfg3", seed=2, T=16, H=512, E=16, W=2)
    for g in range(w.G):
        q, s = oracle.quant_row(w.x_bits[g], mode)
        xf = wl.bf16_bits_to_f32(w.x_bits[g]).astype(np.float64)
        amax = np.abs(xf).max()
        assert s == np.float32(np.float32(amax) / np.float32(127.0 if mode == 2 else 448.0))
        if mode == 2:
            qi = q.view(np.int8).astype(np.float64)
            assert np.abs(qi).max() == 127
            assert np.abs(qi * s - xf).max() <= s / 2 * (1 + 1e-5)
        else:
            deq = np.array([oracle.e4m3_to_f32(int(c)) for c in q], np.float64)
            assert np.abs(deq).max() == 448.0
            v = xf / s
            # half an e4m3 step at |v|: step 2^(floor(log2|v|)-3), at least 2^-9
            e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -6)))
            half = 2.0 ** (e - 3) / 2
            assert (np.abs(deq - v) <= half * (1 + 1e-5) + 1e-6).all()


@pytest.mark.parametrize("seed", range(3))
def test_dispatch_equals_pack_then_exchange(seed):
    """An independent composition: each source rank packs its active slots' token rows in
    stable expert order (numpy argsort), the 1-D exchange plan of the layout's send_splits
    moves them (O1 + O2), and every segment rank d receives from rank r equals expand_x's
    rows of rank d's experts from rank r (O3 + O4) -- the 2-D plan's expert-major order is
    the 1-D exchange regrouped within each receiver."""
    rng = np.random.default_rng(400 + seed)
    W, ne = int(rng.integers(2, 5)), int(rng.integers(1, 4))
    E, T, K, H = W * ne, int(rng.integers(1, 30)), int(rng.integers(1, 4)), 8
    w = wl.moe_workload("tiny", seed=410 + seed, W=W, T=T, K=K, E=E, H=H, active_p=0.8,
                        routing="dup")
    lay = oracle.moe_dispatch_layout(W, T, K, E, w.expert_ids, w.active)
    ex, _, fl = oracle.moe_dispatch(w.x_bits, lay["dst_row"], K, lay["rows_cap"], 0)
    assert fl == 0
    ids = w.expert_ids.reshape(W, T * K)
    act = np.repeat(w.active.astype(bool), K).reshape(W, T * K)
    packs = []
    for r in range(W):
        slots = np.nonzero(act[r])[0]
        order = slots[np.argsort(ids[r][slots], kind="stable")]
        packs.append(w.x_bits[r * T + order // K])
    cap_in = max(1, max(len(pk) for pk in packs))
    inp = np.zeros((W, cap_in, H), np.uint16)
    for r, pk in enumerate(packs):
        inp[r, :len(pk)] = pk
    S = lay["send_splits"]
    src, outs, dsto, _ = oracle.a2a_exchange_plan(S)
    cap_out = max(1, int(outs.sum(axis=1).max()))
    out = np.zeros((W, cap_out, H), np.uint16)
    assert oracle.a2a_v(inp, out, src, outs, dsto) == 0
    cnt, eb = lay["cnt"], lay["expert_base"]
    for d in range(W):
        for r in range(W):
            exp = [ex[eb[e] + cnt[:r, e].sum(): eb[e] + cnt[:r + 1, e].sum()]
                   for e in range(d * ne, (d + 1) * ne)]
            exp = np.concatenate(exp) if exp else np.zeros((0, H), np.uint16)
            got = out[d, dsto[d, r]: dsto[d, r] + outs[d, r]]
            assert np.array_equal(got, exp), (d, r)


def test_dispatch_copy_and_scale_placement():
    w = wl.moe_workload("tiny", seed=4, T=5)
    lay = oracle.moe_dispatch_layout(w.W, w.T, w.K, w.E, w.expert_ids, w.active)
    for mode in (0, 2, 3):
        ex, sc, fl = oracle.moe_dispatch(w.x_bits, lay["dst_row"], w.K, lay["rows_cap"], mode)
        assert fl == 0
        for row in range(lay["R"]):
            g = lay["assist_info"][row] // w.K
            if mode == 0:
                assert (ex[row] == w.x_bits[g]).all()
            else:
                q, s = oracle.quant_row(w.x_bits[g], mode)
                assert (ex[row] == q).all() and sc[row] == s


@pytest.mark.parametrize("mode", [2, 3])
def test_smoothing_brute_force(mode):
    """[P4] scalesOptional: the copy for expert e is x * smooth[e] (fp32 products, here
    numpy's) quantised on its own -- brute force through the independent quantiser."""
    w = wl.moe_workload("tiny", seed=31, W=2, T=6, E=4, K=3, H=48, outlier_frac=0.1,
                        zero_rows=0.1)
    sm = wl.smooth_scales(w.E, w.H, seed=32)
    lay = oracle.moe_dispatch_layout(w.W, w.T, w.K, w.E, w.expert_ids, w.active)
    ex, sc, fl = oracle.moe_dispatch(w.x_bits, lay["dst_row"], w.K, lay["rows_cap"], mode,
                                     smooth=sm, expert_ids=w.expert_ids)
    assert fl == 0
    for row in range(lay["R"]):
        s_ = lay["assist_info"][row]
        g, e = s_ // w.K, w.expert_ids.reshape(-1)[s_]
        xs = wl.bf16_bits_to_f32(w.x_bits[g]).astype(np.float32) * sm[e]
        qb, sb = _quant_brute(xs, mode)
        assert sc[row] == np.float32(sb)
        assert ex[row].tolist() == qb


@pytest.mark.parametrize("mode", [2, 3])
def test_smoothing_special_cases(mode):
    """All-ones smoothing is no smoothing; a power-of-two factor c per expert leaves the
    codes unchanged and multiplies the scale by c exactly."""
    w = wl.moe_workload("tiny", seed=33, W=2, T=10, E=4, K=2, H=64, outlier_frac=0.1)
    lay = oracle.moe_dispatch_layout(w.W, w.T, w.K, w.E, w.expert_ids, w.active)
    plain, psc, _ = oracle.moe_dispatch(w.x_bits, lay["dst_row"], w.K, lay["rows_cap"], mode)
    ones, osc, _ = oracle.moe_dispatch(w.x_bits, lay["dst_row"], w.K, lay["rows_cap"], mode,
                                       smooth=np.ones((w.E, w.H), np.float32),
                                       expert_ids=w.expert_ids)
    assert np.array_equal(plain, ones) and np.array_equal(psc, osc)
    c = np.array([0.25, 2.0, 8.0, 0.5], np.float32)
    pw, pwsc, _ = oracle.moe_dispatch(w.x_bits, lay["dst_row"], w.K, lay["rows_cap"], mode,
                                      smooth=np.repeat(c[:, None], w.H, axis=1),
                                      expert_ids=w.expert_ids)
    assert np.array_equal(pw, plain)
    e_of_row = w.expert_ids.reshape(-1)[lay["assist_info"][:lay["R"]]]
    assert np.array_equal(pwsc[:lay["R"]], psc[:lay["R"]] * c[e_of_row])


def test_smoothing_needs_a_quantising_mode():
    w = wl.moe_workload("tiny", seed=34)
    lay = oracle.moe_dispatch_layout(w.W, w.T, w.K, w.E, w.expert_ids, w.active)
    _, _, fl = oracle.moe_dispatch(w.x_bits, lay["dst_row"], w.K, lay["rows_cap"], 0,
                                   smooth=np.ones((w.E, w.H), np.float32), expert_ids=w.expert_ids)
    assert fl & oracle.ORC_BAD_ARG


# --------------------------------------------------------------- O5 pins

def test_combine_identity_expert_gives_weighted_sum():
    """Identity expert (expert_out = expandX): combine must equal sum_k w[g,k] * x[g]
    computed straight from x, without the layout; with softmax gates it is close to x."""
    w = wl.moe_workload("tiny", seed=8, W=3, T=11, E=9, K=3, H=40)
    lay = oracle.moe_dispatch_layout(w.W, w.T, w.K, w.E, w.expert_ids, w.active)
    ex, _, _ = oracle.moe_dispatch(w.x_bits, lay["dst_row"], w.K, lay["rows_cap"], 0)
    y64, fl = oracle.moe_combine_f64(ex, lay["dst_row"], w.weights, w.K)
    assert fl == 0
    xf = wl.bf16_bits_to_f32(w.x_bits).astype(np.float64)
    wsum = w.weights.astype(np.float64).sum(axis=1)
    assert np.allclose(y64, xf * wsum[:, None], rtol=1e-12, atol=0)
    assert np.abs(y64 - xf).max() <= 1e-6 * np.abs(xf).max() + 1e-6
    y32, _ = oracle.moe_combine_f32(ex, lay["dst_row"], w.weights, w.K)
    yf = wl.bf16_bits_to_f32(y32)
    assert np.allclose(yf, y64, atol=1e-2, rtol=1e-2)


def test_combine_fixed_order_exposes_association():
    """Rows 2^24, +1, -2^24 with unit weights: the fixed k-order fp32 FMA chain gives
    (2^24 + 1) - 2^24 = 0 (2^24+1 rounds to 2^24), while fp64 gives 1; any reordering of
    k changes the fp32 result (the FlashInfer PR's association-order test inputs)."""
    eo = np.array([[wl.f32_to_bf16_bits(np.float32(v))[()] for _ in range(4)]
                   for v in (2.0 ** 24, 1.0, -(2.0 ** 24))], np.uint16)
    w = np.ones((1, 3), np.float32)
    y32, _ = oracle.moe_combine_f32(eo, np.array([0, 1, 2], np.int32), w, 3)
    y64, _ = oracle.moe_combine_f64(eo, np.array([0, 1, 2], np.int32), w, 3)
    assert (wl.bf16_bits_to_f32(y32) == 0).all()
    assert (y64 == 1).all()
    y32b, _ = oracle.moe_combine_f32(eo, np.array([0, 2, 1], np.int32), w, 3)
    assert (wl.bf16_bits_to_f32(y32b) == 1).all()


def test_combine_brute_force_tiny():
    rng = np.random.default_rng(9)
    G, K, H, R = 5, 3, 6, 12
    eo = wl.f32_to_bf16_bits(rng.standard_normal((R, H)).astype(np.float32))
    dr = rng.integers(-1, R, size=(G, K)).astype(np.int32)
    w = rng.random((G, K)).astype(np.float32)
    y64, _ = oracle.moe_combine_f64(eo, dr, w, K)
    y32, _ = oracle.moe_combine_f32(eo, dr, w, K)
    for g in range(G):
        for h in range(H):
            exact = sum(Fraction(float(w[g, k])) * Fraction(float(wl.bf16_bits_to_f32(eo[dr[g, k], h])))
                        for k in range(K) if dr[g, k] >= 0)
            assert abs(y64[g, h] - float(exact)) <= 1e-12 * (1 + abs(float(exact)))
            acc = np.float32(0)
            for k in range(K):
                if dr[g, k] >= 0:
                    # fused multiply-add: exact product + acc, rounded once to fp32
                    p = Fraction(float(w[g, k])) * Fraction(float(wl.bf16_bits_to_f32(eo[dr[g, k], h])))
                    acc = np.float32(_round_f32(p + Fraction(float(acc))))
            ref = torch.tensor([float(acc)], dtype=torch.float32).to(torch.bfloat16)
            assert y32[g, h] == ref.view(torch.int16).numpy().view(np.uint16)[0]
    inactive = (dr < 0).all(axis=1)
    assert (y64[inactive] == 0).all()


def _round_f32(q: Fraction) -> float:
    """Nearest fp32 (ties to even) to an exact rational, by bracketing in fp32."""
    f = float(np.float32(float(q)))          # within an ulp or two
    cands = {f}
    for _ in range(2):
        cands |= {float(np.nextafter(np.float32(c), np.float32(np.inf))) for c in cands}
        cands |= {float(np.nextafter(np.float32(c), np.float32(-np.inf))) for c in cands}
    best = min(cands, key=lambda c: (abs(Fraction(c) - q),
                                     int(np.float32(c).view(np.uint32)) & 1))
    return best


# ----------------------------------------------------- fused tail pins (RMSNorm)

def _rms_case(seed=12, G=6, K=3, H=48, R=20):
    rng = np.random.default_rng(seed)
    eo = wl.f32_to_bf16_bits(rng.standard_normal((R, H)).astype(np.float32))
    dr = rng.integers(-1, R, size=(G, K)).astype(np.int32)
    w = rng.random((G, K)).astype(np.float32)
    res = wl.f32_to_bf16_bits(rng.standard_normal((G, H)).astype(np.float32))
    gamma = (0.5 + rng.random(H)).astype(np.float32)
    return eo, dr, w, res, gamma


def test_rmsnorm_residual_out_brute_force():
    """residual_out = bf16(fp32 FMA chain over k + fp32 residual), by exact rationals."""
    eo, dr, w, res, gamma = _rms_case()
    rout, _, fl = oracle.moe_combine_rmsnorm(eo, dr, w, 3, res, gamma, 1e-6, exact="f32")
    assert fl == 0
    G, H = res.shape
    for g in range(G):
        for h in range(H):
            acc = np.float32(0)
            for k in range(3):
                if dr[g, k] >= 0:
                    p = Fraction(float(w[g, k])) * Fraction(float(wl.bf16_bits_to_f32(eo[dr[g, k], h])))
                    acc = np.float32(_round_f32(p + Fraction(float(acc))))
            s = np.float32(acc) + np.float32(wl.bf16_bits_to_f32(res[g, h]))
            ref = torch.tensor([float(s)], dtype=torch.float32).to(torch.bfloat16)
            assert rout[g, h] == ref.view(torch.int16).numpy().view(np.uint16)[0]


def test_rmsnorm_matches_torch_rms_norm():
    """The normalisation step is torch's rms_norm (a library routine) of residual_out."""
    eo, dr, w, res, gamma = _rms_case(seed=13, G=9, H=64)
    eps = 1e-5
    rout, y64, _ = oracle.moe_combine_rmsnorm(eo, dr, w, 3, res, gamma, eps, exact="f64")
    r = torch.from_numpy(wl.bf16_bits_to_f32(rout).astype(np.float64))
    ref = torch.nn.functional.rms_norm(r, (r.shape[1],), torch.from_numpy(gamma.astype(np.float64)), eps)
    assert np.allclose(y64, ref.numpy(), rtol=1e-12, atol=1e-12)
    rout32, y32, _ = oracle.moe_combine_rmsnorm(eo, dr, w, 3, res, gamma, eps, exact="f32")
    assert np.array_equal(rout32, rout)
    yf = wl.bf16_bits_to_f32(y32).astype(np.float64)
    assert (np.abs(yf - y64) <= 1e-2 + 1e-2 * np.abs(y64)).all()


def test_rmsnorm_closed_form_properties():
    """With gamma = 1 every row's mean square is mean(r^2) / (mean(r^2) + eps); scaling
    gamma scales y; the residual adds exactly into the combined row."""
    eo, dr, w, res, gamma = _rms_case(seed=14, G=5, H=96)
    ones = np.ones_like(gamma)
    eps = 0.25
    rout, y64, _ = oracle.moe_combine_rmsnorm(eo, dr, w, 3, res, ones, eps)
    r = wl.bf16_bits_to_f32(rout).astype(np.float64)
    ms = (r * r).mean(axis=1)
    assert np.allclose((y64 * y64).mean(axis=1), ms / (ms + eps), rtol=1e-12)
    _, y64b, _ = oracle.moe_combine_rmsnorm(eo, dr, w, 3, res, 3.0 * ones, eps)
    assert np.allclose(y64b, 3.0 * y64, rtol=1e-12)
    zero = np.zeros_like(res)
    rz, _, _ = oracle.moe_combine_rmsnorm(eo, dr, w, 3, zero, ones, eps)
    yc, _ = oracle.moe_combine_f64(eo, dr, w, 3)
    assert np.allclose(wl.bf16_bits_to_f32(rz), yc, rtol=2 ** -8, atol=1e-30)


# ------------------------------------------------------------ shared experts

@pytest.mark.parametrize("W,S,N,ne", [(8, 4, 1, 16), (8, 4, 2, 4), (6, 3, 3, 2), (4, 2, 1, 3)])
def test_shared_experts_receive_counts_and_rank_order(W, S, N, ne):
    """[P4]: shared-expert ranks come first (expertShardType 0) and each receives
    Bs * epWorldSize * sharedExpertNum / sharedExpertRankNum tokens; the routed experts
    keep their rows on ranks S..W-1; every token reaches each shared expert once."""
    E = (W - S) * ne
    T, K = 37, 3
    w = wl.moe_workload("tiny", seed=60, W=W, T=T, K=K, E=E)
    ext, extw, E_tot, fl = oracle.shared_expert_routing(W, T, K, E, N, S, w.expert_ids, w.weights)
    assert fl == 0 and E_tot == W * ne
    lay = oracle.moe_dispatch_layout(W, T, K + N, E_tot, ext)
    per_rank = np.diff(lay["rank_base"])
    assert (per_rank[:S] == T * W * N // S).all()
    assert per_rank[S:].sum() == W * T * K
    assert (ext[:, :K] // ne >= S).all() and (ext[:, K:] // ne < S).all()
    # the N shared slots of a token are N different shared experts (replica groups)
    grp = (ext[:, K:] // ne) // (S // N)
    assert all(len(set(row)) == N for row in grp.tolist())
    assert (extw[:, K:] == 1.0).all() and np.array_equal(extw[:, :K], w.weights)
    # routed experts keep their relative order: e -> S*ne + e
    assert np.array_equal(ext[:, :K] - S * ne, w.expert_ids)


def test_shared_experts_identity_expert_combine():
    """Identity experts through the widened routing: y = (sum_k w_k + N) * x."""
    W, S, N, ne, T, K, H = 4, 2, 2, 3, 9, 2, 24
    E = (W - S) * ne
    w = wl.moe_workload("tiny", seed=61, W=W, T=T, K=K, E=E, H=H)
    ext, extw, E_tot, _ = oracle.shared_expert_routing(W, T, K, E, N, S, w.expert_ids, w.weights)
    lay = oracle.moe_dispatch_layout(W, T, K + N, E_tot, ext)
    ex, _, fl = oracle.moe_dispatch(w.x_bits, lay["dst_row"], K + N, lay["rows_cap"], 0)
    y64, fl2 = oracle.moe_combine_f64(ex, lay["dst_row"], extw, K + N)
    assert fl == 0 and fl2 == 0
    xf = wl.bf16_bits_to_f32(w.x_bits).astype(np.float64)
    exp = xf * (w.weights.astype(np.float64).sum(axis=1) + N)[:, None]
    assert np.allclose(y64, exp, rtol=1e-12, atol=1e-12)


def test_shared_experts_argument_rules():
    ids = np.zeros((8, 2), np.int32)
    wts = np.ones((8, 2), np.float32)
    ok = lambda W, E, N, S: oracle.shared_expert_routing(W, 2, 2, E, N, S, ids[:W * 2], wts[:W * 2])[3]
    assert ok(4, 4, 0, 0) == 0                                   # no shared experts
    assert ok(4, 4, 1, 0) & oracle.ORC_BAD_ARG                   # N without shared ranks
    assert ok(4, 4, 2, 1) & oracle.ORC_BAD_ARG                   # S % N != 0
    assert ok(4, 3, 1, 2) & oracle.ORC_BAD_ARG                   # E % (W - S) != 0
    assert ok(4, 4, 1, 3) & oracle.ORC_BAD_ARG                   # W % S != 0
    ext, _, _, _ = oracle.shared_expert_routing(4, 2, 2, 4, 0, 0, ids, wts)
    assert np.array_equal(ext, ids)


@pytest.mark.parametrize("seed", range(6))
def test_layout_segments_are_grouped_by_source_rank(seed):
    """The order the smoothing dispatch may walk rows in rests on this property of the
    layout: within expert e's segment the routed rows come rank by rank, rank r's part
    starting at expert_base[e] + sum_{r'<r} cnt[r'][e] and holding cnt[r][e] rows, and any
    major_align padding follows all of them. Checked on the oracle's layouts (masks,
    duplicates, padding): the parts enumerate every routed row once and each part's rows
    belong to tokens of its rank."""
    rng = np.random.default_rng(700 + seed)
    W = int(rng.integers(1, 9))
    ne = int(rng.integers(1, 6))
    E, K, T = W * ne, int(rng.integers(1, 9)), int(rng.integers(0, 120))
    over = dict(W=W, T=T, K=K, E=E, H=8, routing="dup" if K > E or seed % 2 else "uniform")
    if seed % 3 == 1:
        over["active_p"] = 0.7
    elif seed % 3 == 2:
        over["slot_active_p"] = 0.6
    w = wl.moe_workload("tiny", seed=seed, **over)
    A = [0, 4, 16][seed % 3]
    ref = oracle.moe_dispatch_layout(W, T, K, E, w.expert_ids, w.active, major_align=A)
    cnt, eb, assist = ref["cnt"], ref["expert_base"], ref["assist_info"]
    seen = []
    for e in range(E):
        start = int(eb[e])
        for r in range(W):
            n = int(cnt[r, e])
            rows = np.arange(start, start + n)
            slots = assist[rows]
            assert (slots >= 0).all()
            assert ((slots // K) // T == r).all()               # tokens of rank r
            assert (w.expert_ids.reshape(-1)[slots] == e).all()
            seen.append(rows)
            start += n
        assert (assist[start:int(eb[e + 1])] == -1).all()       # padding after every part
    seen = np.concatenate(seen) if seen else np.zeros(0, np.int64)
    routed = np.nonzero(assist[:ref["R"]] >= 0)[0]
    assert np.array_equal(np.sort(seen), routed)
