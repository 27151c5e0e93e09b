"""Pins for the CPU oracle: checks against facts fixed by the pages and by mathematics.

No test here compares the oracle with itself or retypes its formula: the pins are
hand-worked nibble tables, the worked size examples, exact integer arithmetic with
power-of-two scales, closed forms, the fmt=2 (per-row scale) identity, brute force by
a different algorithm (numpy dense dequantisation + matmul, stable sorting) and
invariants.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from weight_only_int4_gq4_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


# ---------------------------------------------------------------- a1: nibbles
def test_nibble_examples_golden():
    rows = _golden("nibble_examples.txt")
    assert len(rows) >= 10
    for byte, enc, q0, q1 in rows:
        b = int(byte, 16)
        ob = enc == "ob"
        packed = np.array([[b]], np.uint8)
        got = oracle.unpack(packed, 2, offset_binary=ob)[0]
        assert (int(got[0]), int(got[1])) == (int(q0), int(q1)), byte


def test_all_bytes_both_encodings():
    # two's complement nibble n -> ((n ^ 8) - 8); offset binary n -> n - 8
    packed = np.arange(256, dtype=np.uint8)[:, None]
    s4 = oracle.unpack(packed, 2)
    ob = oracle.unpack(packed, 2, offset_binary=True)
    for b in range(256):
        lo, hi = b & 15, b >> 4
        assert s4[b, 0] == ((lo ^ 8) - 8) and s4[b, 1] == ((hi ^ 8) - 8)
        assert ob[b, 0] == lo - 8 and ob[b, 1] == hi - 8


def test_xor_0x88_converts_offset_binary_to_twos_complement():
    packed = np.arange(256, dtype=np.uint8)[:, None]
    assert np.array_equal(oracle.unpack(packed, 2, offset_binary=True),
                          oracle.unpack(packed ^ np.uint8(0x88), 2))


@pytest.mark.parametrize("O,I", [(1, 1), (3, 7), (5, 64), (2, 129), (4, 200)])
@pytest.mark.parametrize("ob", [False, True])
def test_pack_roundtrip_and_pad(O, I, ob):
    q = synth.q_uniform(7, O, I, O, I)
    p = oracle.pack(q, offset_binary=ob)
    assert p.shape == (O, (I + 1) // 2)
    assert np.array_equal(oracle.unpack(p, I, offset_binary=ob), q)
    if I % 2:  # the pad nibble is written as zero
        assert np.all((p[:, -1] >> 4) == 0)


def test_pack_matches_bit_layout():
    # independent bit assembly with numpy: byte = (q_even & 15) | (q_odd & 15) << 4
    q = synth.q_uniform(3, 6, 64)
    ref = ((q[:, 0::2].astype(np.int16) & 15) | ((q[:, 1::2].astype(np.int16) & 15) << 4)).astype(np.uint8)
    assert np.array_equal(oracle.pack(q), ref)


# ---------------------------------------------------------------- sizes
def test_worked_sizes_golden():
    for name, O, I, gs, wb, sb in _golden("sizes.txt"):
        O, I, gs, wb, sb = map(int, (O, I, gs, wb, sb))
        assert oracle.weight_bytes(O, I) == wb, name
        assert oracle.scale_bytes(O, I, gs) == sb, name


def test_expert_size_matches_thread():
    # ~21 MB g64 expert, +2.25 MiB of scales over the per-row (19 MB) expert
    H, F = 6144, 2048
    w = 3 * oracle.weight_bytes(F, H)
    s = 2 * oracle.scale_bytes(F, H, 64) + oracle.scale_bytes(H, F, 64)
    assert w + s == 21233664
    assert s == 2359296 == int(2.25 * 2**20)
    s_row = 2 * oracle.scale_bytes(F, H, H) + oracle.scale_bytes(H, F, F)
    assert 18.8e6 < w + s_row < 19.0e6
    assert abs((w + s) / (w + s_row) - 1.12) < 0.005  # "~12% more resource-hungry"


def test_ngroups_partial():
    assert oracle.ngroups(64, 64) == 1
    assert oracle.ngroups(65, 64) == 2
    assert oracle.ngroups(63, 64) == 1
    assert oracle.ngroups(512, 64) == 8


# ---------------------------------------------------------------- a1-a2: weights, matvec
# The eleven shape classes of the maintainer's oracle test: clean multiples of gs,
# partial last group, odd I, gs > I, gs = 16/64/128, batch, nibble extremes.
SHAPES = [
    (8, 128, 64, 1), (5, 192, 64, 1), (4, 100, 64, 1), (3, 77, 64, 1), (4, 40, 64, 1),
    (6, 96, 16, 1), (6, 256, 128, 1), (7, 130, 128, 1), (5, 128, 64, 4), (3, 33, 16, 3),
    (2, 64, 64, 2),
]


def _pow2_scales(O, ng, seed):
    r = np.random.default_rng(seed)
    return np.ldexp(1.0, r.integers(-9, -2, size=(O, ng))).astype(np.float32) * \
        np.where(r.random((O, ng)) < 0.2, -1, 1).astype(np.float32)


@pytest.mark.parametrize("O,I,gs,T", SHAPES)
def test_matvec_exact_integer_arithmetic(O, I, gs, T):
    """Integer x and power-of-two scales: the exact sum is a small-denominator rational,
    computed here with Python integers from q itself (not from the packed bytes)."""
    q = synth.q_uniform(11, O, I, O, I, gs)
    ng = -(-I // gs)
    s = _pow2_scales(O, ng, O * I + gs)
    r = np.random.default_rng(I)
    x = r.integers(-9, 10, size=(T, I)).astype(np.float32)
    y, bound = oracle.matvec(oracle.pack(q), s, x, gs)
    for t in range(T):
        for o in range(O):
            exact = Fraction(0)
            l1 = Fraction(0)
            for g in range(ng):
                part = sum(int(q[o, k]) * int(x[t, k]) for k in range(g * gs, min(I, (g + 1) * gs)))
                exact += Fraction(float(s[o, g])) * part
                l1 += abs(Fraction(float(s[o, g]))) * sum(abs(int(q[o, k])) for k in range(g * gs, min(I, (g + 1) * gs)))
            assert y[t, o] == float(exact)
            assert bound[t, o] == float(l1 * int(np.abs(x[t]).max()))


@pytest.mark.parametrize("O,I,gs,T", SHAPES)
def test_matvec_vs_numpy_dense(O, I, gs, T):
    """Brute force by another route: numpy dequantises the packed bytes to a dense fp64
    matrix (bit ops on the whole array) and multiplies with np.matmul."""
    q = synth.q_uniform(5, O, I, O, I, gs, 1)
    ng = -(-I // gs)
    s = synth.scales_uniform(5, O, ng, -0.03, 0.03, O, I, gs)
    x = synth.x_normal(5, T, I, "bf16", O, I, gs)
    p = oracle.pack(q)
    b = p.astype(np.int16)
    nib = np.empty((O, 2 * p.shape[1]), np.int16)
    nib[:, 0::2] = b & 15
    nib[:, 1::2] = b >> 4
    qd = np.where(nib >= 8, nib - 16, nib)[:, :I].astype(np.float64)
    W = qd * np.repeat(s.astype(np.float64), gs, axis=1)[:, :I]
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    ref = xf @ W.T
    y, bound = oracle.matvec(p, s, x, gs)
    assert np.all(np.abs(y - ref) <= 1e-12 * bound + 1e-300)


def test_matvec_closed_forms():
    O, I, gs = 4, 256, 64
    r = np.random.default_rng(0)
    x = r.standard_normal((1, I)).astype(np.float32)
    c = np.float32(0.0123)
    # all q = +7, all scales c -> y = 7 c sum(x)
    y, _ = oracle.matvec(np.full((O, I // 2), 0x77, np.uint8), np.full((O, I // gs), c, np.float32), x, gs)
    assert np.allclose(y, 7 * float(c) * x.astype(np.float64).sum(), rtol=1e-13)
    # all q = -8, x = 1 -> y = -8 sum_g s_g len_g (partial last group of 6)
    I2 = 3 * gs + 6
    s = r.uniform(0.1, 1, size=(O, 4)).astype(np.float32)
    y, _ = oracle.matvec(np.full((O, I2 // 2), 0x88, np.uint8), s, np.ones((1, I2), np.float32), gs)
    lens = np.array([gs, gs, gs, 6], np.float64)
    assert np.allclose(y[0], -8 * (s.astype(np.float64) * lens).sum(1), rtol=1e-14)


def test_matvec_one_hot_picks_weight():
    O, I, gs = 9, 320, 64
    q = synth.q_uniform(2, O, I)
    s = synth.scales_uniform(2, O, I // gs, 0.001, 1.0)
    p = oracle.pack(q)
    for k in (0, 1, 63, 64, 65, 200, 319):
        x = np.zeros((1, I), np.float32)
        x[0, k] = 1.0
        y, _ = oracle.matvec(p, s, x, gs)
        assert np.array_equal(y[0], s[:, k // gs].astype(np.float64) * q[:, k])


def test_fmt2_identity_equal_group_scales():
    """All ng scales of a row equal -> the per-row int4 (fmt=2) product s_o * (q . x)."""
    O, I, gs = 7, 384, 64
    q = synth.q_uniform(4, O, I)
    srow = synth.scales_uniform(4, O, 1, 0.002, 0.02)
    s = np.repeat(srow, I // gs, axis=1)
    x = np.random.default_rng(1).integers(-50, 50, size=(2, I)).astype(np.float32)
    y, _ = oracle.matvec(oracle.pack(q), s, x, gs)
    dot = x.astype(np.int64) @ q.astype(np.int64).T  # exact integer per-row dot
    assert np.array_equal(y, dot * srow[:, 0].astype(np.float64)[None, :])
    # and the gs >= I encoding (one group) gives the same numbers
    y1, _ = oracle.matvec(oracle.pack(q), srow, x, I)
    assert np.array_equal(y, y1)


def test_matvec_linearity_and_bound():
    O, I = 16, 512
    q = synth.q_uniform(8, O, I)
    s = synth.scales_uniform(8, O, I // 64, -0.02, 0.02)
    p = oracle.pack(q)
    r = np.random.default_rng(3)
    x1 = r.standard_normal((1, I)).astype(np.float32)
    x2 = r.standard_normal((1, I)).astype(np.float32)
    y1, b1 = oracle.matvec(p, s, x1)
    y2, _ = oracle.matvec(p, s, x2)
    y12, _ = oracle.matvec(p, s, x1 + x2)  # x1+x2 rounded to f32: compare loosely
    assert np.allclose(y12, y1 + y2, atol=1e-5 * b1.max())
    assert np.all(np.abs(y1) <= b1)


# ---------------------------------------------------------------- bf16 rounding
def test_round_bf16_hand_cases():
    assert oracle.round_bf16(1.0 + 2**-8) == 1.0            # tie -> even
    assert oracle.round_bf16(1.0 + 3 * 2**-8) == 1.0 + 2**-6  # tie -> even (up)
    assert oracle.round_bf16(1.0 + 2**-8 + 2**-30) == 1.0 + 2**-7
    assert oracle.round_bf16(-3.0) == -3.0
    assert oracle.round_bf16(0.0) == 0.0
    assert math.isinf(oracle.round_bf16(3.4e38))
    assert oracle.round_bf16(2.0**-133) == 2.0**-133         # smallest bf16 subnormal
    assert oracle.round_bf16(2.0**-135) == 0.0


def test_round_bf16_matches_integer_rne_on_f32_values():
    v = np.random.default_rng(5).standard_normal(20000).astype(np.float32) * 100
    ref = synth.bf16_bits_to_f32(synth.to_bf16_bits(v)).astype(np.float64)
    got = np.array([oracle.round_bf16(float(a)) for a in v])
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------- a3: gate/up/SiLU
def test_gate_up_pair_invariant_and_silu():
    F, H = 32, 256
    qg, qu = synth.q_uniform(1, F, H, 0), synth.q_uniform(1, F, H, 1)
    sg = synth.scales_uniform(1, F, H // 64, 0.005, 0.02, 0)
    su = synth.scales_uniform(1, F, H // 64, 0.005, 0.02, 1)
    x = synth.x_normal(1, 3, H, "f32")
    pg, pu = oracle.pack(qg), oracle.pack(qu)
    h, g, u = oracle.gate_up_silu(pg, sg, pu, su, x)
    # pair(g,u) == grouped(g), grouped(u), elementwise
    assert np.array_equal(g, oracle.matvec(pg, sg, x)[0])
    assert np.array_equal(u, oracle.matvec(pu, su, x)[0])
    # SiLU on the gate side, not on up: h/u = g*sigmoid(g), monotone limits
    ratio = h / u
    sig = 1 / (1 + np.exp(-g))
    assert np.allclose(ratio, g * sig, rtol=1e-6)
    assert np.all((np.sign(h) == np.sign(g * u)) | (h == 0))


def test_silu_special_values():
    # one-hot x isolates one weight: g = s_g q_g, u = s_u q_u exactly
    F, H = 4, 64
    qg = np.zeros((F, H), np.int8)
    qu = np.zeros((F, H), np.int8)
    qg[:, 5] = [0, 7, -8, 1]
    qu[:, 5] = [3, 2, 5, -4]
    sg = np.array([[1.0], [8.0], [8.0], [0.5]], np.float32)
    su = np.ones((F, 1), np.float32)
    x = np.zeros((1, H), np.float32)
    x[0, 5] = 1.0
    h, g, u = oracle.gate_up_silu(oracle.pack(qg), sg, oracle.pack(qu), su, x)
    assert h[0, 0] == 0.0                                  # silu(0) = 0
    assert abs(h[0, 1] - 56.0 * 2) < 56 * 2 * 1e-20 + 1e-9  # g = 56 >> 0: h ~ g*u
    assert -1e-20 < h[0, 2] <= 0.0                         # g = -64 << 0: h -> 0 from below
    assert np.float32(h[0, 3]) == np.float32(0.5 / (1 + math.exp(-0.5)) * -4)


def test_gate_up_bf16_output_is_rounded():
    F, H = 16, 128
    pg = oracle.pack(synth.q_uniform(9, F, H, 0))
    pu = oracle.pack(synth.q_uniform(9, F, H, 1))
    s = synth.scales_uniform(9, F, 2, 0.005, 0.02)
    x = synth.x_normal(9, 2, H, "bf16")
    h, g, u = oracle.gate_up_silu(pg, s, pu, s, x)
    hb = synth.bf16_bits_to_f32(synth.to_bf16_bits(h.astype(np.float32))).astype(np.float64)
    assert np.array_equal(h, hb)  # every value is a bf16 number
    exact = g / (1 + np.exp(-g)) * u
    assert np.all(np.abs(h - exact) <= np.abs(exact) * 2**-8 * 1.0000001)


# ---------------------------------------------------------------- a4: router
def test_route_matches_stable_sort_and_subset_softmax():
    T, E, K = 50, 64, 8
    lg, _ = synth.logits_normal(3, T, E)
    st, idx, wts, bad = oracle.route(lg, K)
    assert st == oracle.OK and not bad.any()
    order = np.argsort(-lg.astype(np.float64), axis=1, kind="stable")[:, :K]
    assert np.array_equal(idx, order)
    sel = np.take_along_axis(lg.astype(np.float64), order, 1)
    sm = np.exp(sel - sel.max(1, keepdims=True))
    sm /= sm.sum(1, keepdims=True)
    assert np.allclose(wts, sm, rtol=1e-13, atol=0)
    assert np.allclose(wts.sum(1), 1.0, atol=1e-14)
    assert np.all(np.diff(wts, axis=1) <= 0)


def test_route_ties_and_edges():
    lg = np.array([[1, 3, 3, 0, 3, -1], [0, 0, 0, 0, 0, 0]], np.float32)
    st, idx, wts, bad = oracle.route(lg, 3)
    assert idx.tolist() == [[1, 2, 4], [0, 1, 2]]
    assert np.allclose(wts, 1 / 3, rtol=1e-15)
    st, idx, wts, _ = oracle.route(lg, 6)  # K = E: every expert, descending logit
    assert idx[0].tolist() == [1, 2, 4, 0, 3, 5]
    st, idx, wts, _ = oracle.route(lg[:1], 1)  # K = 1: weight 1
    assert idx.tolist() == [[1]] and wts[0, 0] == 1.0
    st, idx, wts, _ = oracle.route(np.array([[-np.inf, 2, -np.inf, 1]], np.float32), 3)
    assert idx.tolist() == [[1, 3, 0]] and wts[0, 2] == 0.0


def test_route_rejects_nonfinite():
    lg = np.zeros((3, 8), np.float32)
    lg[1, 4] = np.nan
    lg[2, :] = -np.inf
    st, idx, wts, bad = oracle.route(lg, 2)
    assert st == oracle.ERR_NONFINITE_LOGIT
    assert bad.tolist() == [0, 1, 1]
    assert np.all(np.isnan(wts[1:])) and np.all(np.isfinite(wts[0]))
    lg = np.zeros((1, 8), np.float32)
    lg[0, 0] = np.inf
    assert oracle.route(lg, 2)[0] == oracle.ERR_NONFINITE_LOGIT


# ---------------------------------------------------------------- a5: row map
@pytest.mark.parametrize("T,E,K", [(1, 128, 8), (32, 256, 8), (7, 4, 4), (100, 16, 2), (3, 5, 1)])
def test_rowmap_vs_stable_argsort(T, E, K):
    idx = np.stack([np.random.default_rng(T + t).permutation(E)[:K] for t in range(T)]).astype(np.int32)
    m = oracle.rowmap(idx, E)
    flat = idx.reshape(-1)
    assert np.array_equal(m["cnt"], np.bincount(flat, minlength=E))
    assert m["offs"][0] == 0 and m["offs"][-1] == T * K and np.all(np.diff(m["offs"]) >= 0)
    order = np.argsort(flat, kind="stable")  # rows grouped by expert, slots ascending
    assert np.array_equal(m["row_slot"], order)
    assert np.array_equal(m["row_tok"], order // K)
    assert np.array_equal(m["slot_row"][m["row_slot"]], np.arange(T * K))
    for e in range(E):
        seg = m["row_slot"][m["offs"][e]:m["offs"][e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)


# ---------------------------------------------------------------- row L1 norms (tolerance scale)
# The per-element acceptance bound is 2e-3 * ||w_row||_1 * max|x| ("compare against the
# sum of |terms|", the maintainer's oracle reply on colibri PR #298); these pins fix the
# norm the bound is built from.
def _dense_any(p, s, I, gs):
    """Independent numpy decode for any group size and odd widths (low nibble first,
    two's complement, scale of column k = s[:, k // gs])."""
    b = p.astype(np.int16)
    nib = np.empty((p.shape[0], 2 * p.shape[1]), np.int16)
    nib[:, 0::2] = b & 15
    nib[:, 1::2] = b >> 4
    q = np.where(nib >= 8, nib - 16, nib)[:, :I].astype(np.float64)
    cols = np.arange(I) // gs
    return q * s.astype(np.float64)[:, cols]


@pytest.mark.parametrize("O,I,gs", [(7, 64, 64), (5, 200, 64), (3, 129, 16), (4, 96, 128),
                                    (6, 33, 64), (2, 512, 64), (9, 250, 48)])
def test_row_l1_vs_numpy_dense(O, I, gs):
    r = np.random.default_rng(O * 1000 + I)
    q = r.integers(-8, 8, size=(O, I)).astype(np.int8)
    ng = -(-I // gs)
    # signed scales: the norm is over |s * q|, so a negative scale must count positively
    s = (r.uniform(0.002, 0.02, size=(O, ng)) * r.choice([-1.0, 1.0], size=(O, ng))).astype(np.float32)
    p = oracle.pack(q)
    got = oracle.row_l1(p, s, I, gs)
    want = np.abs(_dense_any(p, s, I, gs)).sum(1)
    assert np.allclose(got, want, rtol=1e-12, atol=0)
    # the matvec's own bound is the same norm times max|x| of each token
    x = r.standard_normal((2, I)).astype(np.float32)
    _, b = oracle.matvec(p, s, x, gs)
    assert np.allclose(b, want[None, :] * np.abs(x).max(1)[:, None], rtol=1e-12, atol=0)


def test_row_l1_exact_power_of_two_scales():
    """Hand-worked norms with scales 2^-j, exact in fp64: a row of all -8 over 3 groups,
    an alternating +7/-8 row, a row of zeros, and a row whose second group is the only
    nonzero one (catches a norm summed over the wrong axis or without |.|)."""
    I, gs = 192, 64
    q = np.zeros((4, I), np.int8)
    q[0] = -8
    q[1, 0::2], q[1, 1::2] = 7, -8
    q[3, 64:128] = 3
    s = np.array([[2.0 ** -3, 2.0 ** -4, 2.0 ** -5],
                  [-2.0 ** -2, 2.0 ** -2, -2.0 ** -2],
                  [1.0, 1.0, 1.0],
                  [2.0 ** -7, -2.0 ** -6, 2.0 ** -7]], np.float32)
    got = oracle.row_l1(oracle.pack(q), s, I, gs)
    want = [8 * 64 * (2.0 ** -3 + 2.0 ** -4 + 2.0 ** -5),
            (7 + 8) * 32 * 3 * 2.0 ** -2,
            0.0,
            3 * 64 * 2.0 ** -6]
    assert list(got) == want


# ---------------------------------------------------------------- a6-a8: MoE
def _dense(p, s, I, gs=64):
    b = p.astype(np.int16)
    nib = np.empty((p.shape[0], 2 * p.shape[1]), np.int16)
    nib[:, 0::2] = b & 15
    nib[:, 1::2] = b >> 4
    q = np.where(nib >= 8, nib - 16, nib)[:, :I].astype(np.float64)
    return q * np.repeat(s.astype(np.float64), gs, axis=1)[:, :I]


def _toy_moe(E=4, K=2, H=128, F=128, T=5, seed=21):
    pg = np.stack([synth.packed_uniform(seed, F, H, 0, e) for e in range(E)])
    pu = np.stack([synth.packed_uniform(seed, F, H, 1, e) for e in range(E)])
    pd = np.stack([synth.packed_uniform(seed, H, F, 2, e) for e in range(E)])
    sg = np.stack([synth.scales_uniform(seed, F, H // 64, 0.002, 0.02, 0, e) for e in range(E)])
    su = np.stack([synth.scales_uniform(seed, F, H // 64, 0.002, 0.02, 1, e) for e in range(E)])
    sd = np.stack([synth.scales_uniform(seed, H, F // 64, 0.002, 0.02, 2, e) for e in range(E)])
    x = synth.x_normal(seed, T, H, "bf16")
    lg, _ = synth.logits_normal(seed, T, E)
    return pg, sg, pu, su, pd, sd, x, lg


def test_moe_bruteforce_numpy_dense():
    E, K, H, F, T = 4, 2, 128, 128, 5
    pg, sg, pu, su, pd, sd, x, lg = _toy_moe(E, K, H, F, T)
    st, idx, wts, _ = oracle.route(lg, K)
    y, bound = oracle.moe_tokens(pg, sg, pu, su, pd, sd, H, F, x, idx, wts, np.arange(T))
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    for t in range(T):
        acc = np.zeros(H)
        for j in range(K):
            e = idx[t, j]
            g = _dense(pg[e], sg[e], H) @ xf[t]
            u = _dense(pu[e], su[e], H) @ xf[t]
            h = g / (1 + np.exp(-g)) * u
            hb = synth.bf16_bits_to_f32(synth.to_bf16_bits(h.astype(np.float32))).astype(np.float64)
            acc += wts[t, j] * (_dense(pd[e], sd[e], F) @ hb)
        # rare f64->f32->bf16 double roundings differ by one bf16 ulp of one h element
        assert np.all(np.abs(y[t] - acc) <= 1e-4 * bound[t])
        assert np.all(np.abs(y[t]) <= bound[t])


def test_moe_reduces_to_single_expert():
    """T=1, K=E=1, weight 1: the MoE layer is down(gate_up_silu(x))."""
    H, F = 128, 192
    pg, sg, pu, su, pd, sd, x, _ = _toy_moe(1, 1, H, F, 1, seed=4)
    st, idx, wts, _ = oracle.route(np.zeros((1, 1), np.float32), 1)
    assert idx[0, 0] == 0 and wts[0, 0] == 1.0
    y, _ = oracle.moe_tokens(pg, sg, pu, su, pd, sd, H, F, x, idx, wts, np.arange(1))
    h, _, _ = oracle.gate_up_silu(pg[0], sg[0], pu[0], su[0], x)
    hb = synth.to_bf16_bits(h.astype(np.float32))  # h is already bf16-valued: exact
    y1, _ = oracle.matvec(pd[0], sd[0], hb)
    assert np.array_equal(y, y1)
