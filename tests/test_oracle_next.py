"""Pins for the oracle functions of the NEXT rows: group-size detection, quantisation,
row dequantisation / gather and the matvec over selected rows.

As in test_oracle.py, nothing here compares the oracle with itself: the pins are the
pages' worked sizes, hand-worked rounding examples, exact round trips on values that lie
on the quantisation grid, closed-form error bounds and invariants, and an independent
numpy decode of the packed bytes (the closed form ((n ^ 8) - 8) pinned by the nibble
tables) with a dense matmul.
"""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
CANDIDATES = (16, 32, 48, 64, 96, 128, 192, 256)


def _golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


def _np_dequant(packed, scales, I, gs):
    """Independent decode: low nibble first, two's complement ((n ^ 8) - 8), scale per group."""
    O = packed.shape[0]
    lo = (packed & 15).astype(np.int64)
    hi = (packed >> 4).astype(np.int64)
    q = np.empty((O, 2 * packed.shape[1]), np.int64)
    q[:, 0::2] = (lo ^ 8) - 8
    q[:, 1::2] = (hi ^ 8) - 8
    q = q[:, :I]
    g = np.arange(I) // gs
    return scales.astype(np.float64)[:, g] * q


# ---------------------------------------------------------------- detect_group_size
def test_detect_group_size_worked_sizes():
    for name, O, I, gs, wb, sb in _golden("sizes.txt"):
        O, I, gs, sb = int(O), int(I), int(gs), int(sb)
        got = oracle.detect_group_size(O, I, sb)
        if gs in CANDIDATES:
            assert got == gs, name
        else:  # per-row scales: no candidate gives one group per row at these widths
            assert got == 0, name


def test_detect_group_size_gs128_and_edges():
    # the pages validate a gs=128 conversion of the same expert shapes
    assert oracle.detect_group_size(2048, 6144, 2048 * (6144 // 128) * 4) == 128
    assert oracle.detect_group_size(6144, 2048, 6144 * (2048 // 128) * 4) == 128
    assert oracle.detect_group_size(100, 4096, 123) == 0            # no candidate
    assert oracle.detect_group_size(100, 16, 100 * 4) == -1          # every candidate: 1 group


@pytest.mark.parametrize("I", [48, 96, 640, 1000, 4096, 6144, 7168])
def test_detect_group_size_brute_force(I):
    """Every candidate either is recovered from its own scale size or collides with
    another candidate giving the same number of groups (then the answer is -1)."""
    for gs in CANDIDATES:
        ng = -(-I // gs)
        same = [c for c in CANDIDATES if -(-I // c) == ng]
        got = oracle.detect_group_size(3, I, 3 * ng * 4)
        assert got == (gs if len(same) == 1 else -1)


# ---------------------------------------------------------------- quantize
def test_quantize_hand_examples():
    for row in _golden("quantize_examples.txt"):
        s_expect = float(row[0])
        pairs = [p.split(":") for p in row[1:]]
        w = np.array([[float(a) for a, _ in pairs]], np.float32)
        q_expect = [int(b) for _, b in pairs]
        q, s = oracle.quantize(w, gs=8)
        assert s.shape == (1, 1) and float(s[0, 0]) == s_expect
        assert q[0].tolist() == q_expect


@pytest.mark.parametrize("O,I,gs", [(5, 64, 64), (3, 200, 64), (4, 256, 32), (2, 96, 48), (3, 130, 16),
                                    (2, 512, 128)])
def test_quantize_exact_round_trip_on_grid(O, I, gs):
    """w = c * q with c a power of two and a +-7 in every group: quantize returns q and c."""
    rng = np.random.default_rng(O * 1000 + I)
    ng = -(-I // gs)
    q = rng.integers(-7, 8, size=(O, I))
    c = 2.0 ** rng.integers(-12, 6, size=(O, ng))
    for o in range(O):
        for g in range(ng):
            q[o, g * gs + rng.integers(0, min(gs, I - g * gs))] = rng.choice([-7, 7])
    w = (c[:, np.arange(I) // gs] * q).astype(np.float32)
    qq, s = oracle.quantize(w, gs)
    assert np.array_equal(qq, q.astype(np.int8))
    assert np.array_equal(s, c.astype(np.float32))


@pytest.mark.parametrize("gs", [16, 64, 128])
def test_quantize_error_bound_and_invariants(gs):
    rng = np.random.default_rng(gs)
    O, I = 7, 384
    w = (rng.standard_normal((O, I)) * rng.uniform(0.01, 3.0, size=(O, 1))).astype(np.float32)
    w[2, :gs] = 0.0  # an all-zero group
    q, s = oracle.quantize(w, gs)
    ng = I // gs
    g = np.arange(I) // gs
    # |w - s*q| <= s/2 (no clamping happens: |w/s| <= 7), up to one f32 rounding of w/s
    err = np.abs(w.astype(np.float64) - s.astype(np.float64)[:, g] * q)
    assert np.all(err <= s.astype(np.float64)[:, g] * (0.5 + 1e-6))
    assert q.min() >= -7 and q.max() <= 7  # -8 never occurs with s = max|w| / 7
    for o in range(O):
        for gg in range(ng):
            blk = w[o, gg * gs:(gg + 1) * gs]
            qb = q[o, gg * gs:(gg + 1) * gs]
            if not np.any(blk):
                assert s[o, gg] == 0 and not np.any(qb)
                continue
            assert np.abs(qb).max() == 7
            assert abs(int(qb[np.argmax(np.abs(blk))])) == 7
    # sign symmetry and power-of-two scale invariance
    q2, s2 = oracle.quantize(-w, gs)
    assert np.array_equal(q2, -q) and np.array_equal(s2, s)
    q3, s3 = oracle.quantize(w * np.float32(8.0), gs)
    assert np.array_equal(q3, q) and np.array_equal(s3, s * np.float32(8.0))


def test_quantize_per_row_is_fmt2():
    rng = np.random.default_rng(5)
    w = rng.standard_normal((4, 100)).astype(np.float32)
    q, s = oracle.quantize(w, gs=100)
    assert s.shape == (4, 1)
    assert np.array_equal(s[:, 0], (np.abs(w).max(1) / np.float32(7.0)).astype(np.float32))


# ---------------------------------------------------------------- row ops
@pytest.mark.parametrize("O,I,gs", [(9, 256, 64), (6, 200, 64), (5, 96, 32), (4, 130, 128)])
def test_dequant_rows_vs_numpy(O, I, gs):
    rng = np.random.default_rng(I + gs)
    q = rng.integers(-8, 8, size=(O, I)).astype(np.int8)
    s = rng.uniform(-0.02, 0.02, size=(O, -(-I // gs))).astype(np.float32)
    p = oracle.pack(q)
    idx = rng.integers(0, O, size=7).astype(np.int32)
    dense = _np_dequant(p, s, I, gs)
    assert np.array_equal(oracle.dequant_rows(p, s, I, idx, gs), dense[idx])
    alpha = rng.standard_normal(7)
    base = rng.standard_normal((7, I))
    got = oracle.dequant_rows(p, s, I, idx, gs, alpha=alpha, out=base)
    assert np.allclose(got, base + alpha[:, None] * dense[idx], rtol=0, atol=1e-15)


@pytest.mark.parametrize("O,I,gs,T", [(12, 256, 64, 1), (8, 200, 64, 3), (6, 96, 32, 2), (5, 130, 16, 1)])
def test_matvec_rows_vs_numpy(O, I, gs, T):
    rng = np.random.default_rng(O * I + T)
    q = rng.integers(-8, 8, size=(O, I)).astype(np.int8)
    s = rng.uniform(-0.02, 0.02, size=(O, -(-I // gs))).astype(np.float32)
    p = oracle.pack(q)
    idx = np.array([O - 1, 0, 3, 3, 1], np.int32)
    x = rng.standard_normal((T, I)).astype(np.float32)
    y, b = oracle.matvec_rows(p, s, idx, x, gs)
    dense = _np_dequant(p, s, I, gs)
    ref = x.astype(np.float64) @ dense[idx].T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    assert np.all(np.abs(y) <= b * (1 + 1e-12))


# ---------------------------------------------------------------- MLA absorb projections
def _mla_tensor(nh, dn, dv, R, gs, seed, pow2=False):
    """kv_b-like tensor: nh blocks of dn key rows + dv value rows, R inputs."""
    rng = np.random.default_rng(seed)
    O = nh * (dn + dv)
    q = rng.integers(-8, 8, size=(O, R)).astype(np.int8)
    ng = -(-R // gs)
    if pow2:
        scales = (2.0 ** rng.integers(-6, 2, size=(O, ng))).astype(np.float32)
    else:
        scales = rng.uniform(0.002, 0.02, size=(O, ng)).astype(np.float32)
    return q, oracle.pack(q), scales


@pytest.mark.parametrize("nh,dn,dv,R,gs,T", [(2, 3, 5, 128, 64, 1), (3, 16, 8, 96, 64, 2),
                                             (1, 4, 4, 40, 16, 3), (2, 8, 16, 512, 64, 2)])
def test_mla_absorb_vs_numpy(nh, dn, dv, R, gs, T):
    """Both projections against an independent decode and einsum over the head blocks
    (partial last group in the 96- and 40-wide cases)."""
    _, packed, scales = _mla_tensor(nh, dn, dv, R, gs, seed=nh * 100 + R)
    W = _np_dequant(packed, scales, R, gs).reshape(nh, dn + dv, R)
    rng = np.random.default_rng(R)
    qn = rng.standard_normal((T, nh, dn)).astype(np.float32)
    lat = rng.standard_normal((T, nh, R)).astype(np.float32)
    got_q, b_q = oracle.mla_absorb_q(packed, scales, R, nh, dn, dv, qn, gs)
    ref_q = np.einsum("thd,hdc->thc", qn.astype(np.float64), W[:, :dn, :])
    np.testing.assert_allclose(got_q, ref_q, rtol=1e-12, atol=1e-12 * np.abs(ref_q).max())
    assert np.all(np.abs(ref_q) <= b_q * (1 + 1e-12))
    got_v, b_v = oracle.mla_absorb_v(packed, scales, R, nh, dn, dv, lat, gs)
    ref_v = np.einsum("thc,hvc->thv", lat.astype(np.float64), W[:, dn:, :])
    np.testing.assert_allclose(got_v, ref_v, rtol=1e-12, atol=1e-12 * np.abs(ref_v).max())
    assert np.all(np.abs(ref_v) <= b_v * (1 + 1e-12))


def test_mla_absorb_exact_integer_arithmetic():
    """Power-of-two scales and integer inputs: every product and partial sum is exact in
    fp64, so the results equal integer arithmetic done in Python."""
    nh, dn, dv, R, gs, T = 2, 5, 3, 80, 16, 2
    q, packed, scales = _mla_tensor(nh, dn, dv, R, gs, seed=5, pow2=True)
    rng = np.random.default_rng(6)
    qn = rng.integers(-4, 5, size=(T, nh, dn)).astype(np.float32)
    lat = rng.integers(-4, 5, size=(T, nh, R)).astype(np.float32)
    got_q, _ = oracle.mla_absorb_q(packed, scales, R, nh, dn, dv, qn, gs)
    got_v, _ = oracle.mla_absorb_v(packed, scales, R, nh, dn, dv, lat, gs)
    D = dn + dv
    for t in range(T):
        for h in range(nh):
            for c in range(R):
                want = sum(int(qn[t, h, d]) * int(q[h * D + d, c]) * float(scales[h * D + d, c // gs])
                           for d in range(dn))
                assert got_q[t, h, c] == want
            for v in range(dv):
                r = h * D + dn + v
                want = sum(int(lat[t, h, c]) * int(q[r, c]) * float(scales[r, c // gs]) for c in range(R))
                assert got_v[t, h, v] == want


def test_mla_absorb_q_one_hot_reads_the_group_scale():
    """A one-hot q_nope on (head h, key row d) returns that kv_b row exactly, with the
    scale of each column's own group; one scale per row (the fmt=2 rule the pages' crash
    came from) gives a different row."""
    nh, dn, dv, R, gs = 3, 4, 2, 256, 64
    q, packed, scales = _mla_tensor(nh, dn, dv, R, gs, seed=9, pow2=True)
    scales[:, 1] *= 2.0  # make sure neighbouring groups of a row differ
    h, d = 2, 3
    row = h * (dn + dv) + d
    qn = np.zeros((1, nh, dn), np.float32)
    qn[0, h, d] = 1.0
    got, _ = oracle.mla_absorb_q(packed, scales, R, nh, dn, dv, qn, gs)
    want = scales[row, np.arange(R) // gs].astype(np.float64) * q[row].astype(np.float64)
    assert np.array_equal(got[0, h], want)
    assert not np.any(got[0, [0, 1]])
    per_row = scales.reshape(-1)[row] * q[row].astype(np.float64)  # wscale[row] on an O*ng buffer
    assert not np.array_equal(got[0, h], per_row)


def test_mla_absorb_v_one_hot_and_fmt2_identity():
    """A one-hot latent channel c returns column c of each head's value rows; with all
    group scales of a row equal, the V projection is the per-row (fmt=2) product."""
    nh, dn, dv, R, gs = 2, 3, 4, 128, 64
    q, packed, scales = _mla_tensor(nh, dn, dv, R, gs, seed=11, pow2=True)
    c = 77
    lat = np.zeros((1, nh, R), np.float32)
    lat[0, :, c] = 1.0
    got, _ = oracle.mla_absorb_v(packed, scales, R, nh, dn, dv, lat, gs)
    D = dn + dv
    for h in range(nh):
        rows = h * D + dn + np.arange(dv)
        assert np.array_equal(got[0, h], scales[rows, c // gs].astype(np.float64) * q[rows, c])
    flat = np.repeat(scales[:, :1], scales.shape[1], axis=1)  # one scale per row
    rng = np.random.default_rng(12)
    lat = rng.integers(-3, 4, size=(2, nh, R)).astype(np.float32)
    got, _ = oracle.mla_absorb_v(packed, flat, R, nh, dn, dv, lat, gs)
    for h in range(nh):
        rows = h * D + dn + np.arange(dv)
        want = flat[rows, 0].astype(np.float64)[None] * (lat[:, h].astype(np.int64) @ q[rows].T.astype(np.int64))
        assert np.array_equal(got[:, h], want)
