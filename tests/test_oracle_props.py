"""Property-based pins of the oracle (hypothesis, CPU only): on random small shapes each
function is checked against an independent formulation -- a numpy decode + matmul for
the grouped products, a stable sort + subset softmax for the router, argsort/bincount
for the row map, the per-row identity for equal group scales -- so a dropped term, a
wrong index or a swapped operand anywhere in the oracle fails one of them."""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle

# derandomized: the same examples every run, so the suite is reproducible
SETTINGS = settings(max_examples=40, deadline=None, derandomize=True, suppress_health_check=[HealthCheck.too_slow])


def _decode(packed, scales, I, gs):
    lo = (packed & 15).astype(np.int64)
    hi = (packed >> 4).astype(np.int64)
    q = np.empty((packed.shape[0], 2 * packed.shape[1]), np.int64)
    q[:, 0::2] = (lo ^ 8) - 8
    q[:, 1::2] = (hi ^ 8) - 8
    q = q[:, :I]
    return scales.astype(np.float64)[:, np.arange(I) // gs] * q


@SETTINGS
@given(O=st.integers(1, 12), I=st.integers(1, 70), gs=st.sampled_from([8, 16, 32, 64, 128]),
       T=st.integers(1, 3), seed=st.integers(0, 2**31 - 1))
def test_matvec_matches_numpy_decode(O, I, gs, T, seed):
    rng = np.random.default_rng(seed)
    packed = rng.integers(0, 256, size=(O, (I + 1) // 2), dtype=np.uint8)
    if I % 2:
        packed[:, -1] &= 15  # the pad nibble of an odd row is written as 0
    scales = rng.uniform(-0.05, 0.05, size=(O, -(-I // gs))).astype(np.float32)
    x = rng.standard_normal((T, I)).astype(np.float32)
    y, b = oracle.matvec(packed, scales, x, gs)
    ref = x.astype(np.float64) @ _decode(packed, scales, I, gs).T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12 * (np.abs(ref).max() + 1))
    assert np.all(np.abs(ref) <= b * (1 + 1e-12) + 1e-300)


@SETTINGS
@given(O=st.integers(1, 8), I=st.sampled_from([8, 24, 64, 100]), gs=st.sampled_from([8, 32, 64]),
       seed=st.integers(0, 2**31 - 1))
def test_equal_group_scales_reduce_to_per_row(O, I, gs, seed):
    rng = np.random.default_rng(seed)
    q = rng.integers(-8, 8, size=(O, I)).astype(np.int8)
    packed = oracle.pack(q)
    s_row = (2.0 ** rng.integers(-4, 3, size=O)).astype(np.float32)
    scales = np.repeat(s_row[:, None], -(-I // gs), axis=1)
    x = rng.integers(-3, 4, size=(2, I)).astype(np.float32)
    y, _ = oracle.matvec(packed, scales, x, gs)
    want = (x.astype(np.int64) @ q.T.astype(np.int64)) * s_row.astype(np.float64)[None]
    assert np.array_equal(y, want)


@SETTINGS
@given(T=st.integers(1, 6), E=st.integers(1, 40), data=st.data())
def test_router_matches_stable_sort_and_subset_softmax(T, E, data):
    K = data.draw(st.integers(1, E))
    seed = data.draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    lg = rng.integers(-3, 4, size=(T, E)).astype(np.float32)  # many ties
    status, idx, wts, bad = oracle.route(lg, K)
    assert status == 0 and not bad.any()
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(lg[t, e]), e))[:K]
        assert list(idx[t]) == order
        sel = lg[t, order].astype(np.float64)
        p = np.exp(sel - sel.max())
        np.testing.assert_allclose(wts[t], p / p.sum(), rtol=1e-12)


@SETTINGS
@given(T=st.integers(1, 20), E=st.integers(1, 12), data=st.data())
def test_rowmap_matches_argsort_and_bincount(T, E, data):
    K = data.draw(st.integers(1, E))
    seed = data.draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    m = oracle.rowmap(idx, E)
    flat = idx.reshape(-1)
    assert np.array_equal(m["cnt"], np.bincount(flat, minlength=E))
    order = np.argsort(flat, kind="stable")
    assert np.array_equal(m["row_slot"], order)
    assert np.array_equal(m["row_tok"], order // K)
    assert np.array_equal(m["slot_row"][m["row_slot"]], np.arange(T * K))
    assert np.array_equal(m["offs"], np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))


@settings(max_examples=15, deadline=None, derandomize=True, suppress_health_check=[HealthCheck.too_slow])
@given(E=st.integers(1, 5), T=st.integers(1, 4), H=st.sampled_from([64, 128]), F=st.sampled_from([64, 192]),
       data=st.data())
def test_moe_layer_matches_dense_brute_force(E, T, H, F, data):
    """The whole layer on random small configurations against a dense numpy evaluation
    of its definition: route, then per slot silu(g)*u rounded to bf16, down, weighted."""
    K = data.draw(st.integers(1, E))
    seed = data.draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    pg = rng.integers(0, 256, size=(E, F, H // 2), dtype=np.uint8)
    pu = rng.integers(0, 256, size=(E, F, H // 2), dtype=np.uint8)
    pd = rng.integers(0, 256, size=(E, H, F // 2), dtype=np.uint8)
    sg = rng.uniform(0.002, 0.02, size=(E, F, H // 64)).astype(np.float32)
    su = rng.uniform(0.002, 0.02, size=(E, F, H // 64)).astype(np.float32)
    sd = rng.uniform(0.002, 0.02, size=(E, H, F // 64)).astype(np.float32)
    xf32 = rng.standard_normal((T, H)).astype(np.float32)
    x = (xf32.view(np.uint32) >> 16).astype(np.uint16)  # bf16 bits (truncated: any bf16 values will do)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    status, idx, wts, _ = oracle.route(lg, K)
    y, bound = oracle.moe_tokens(pg, sg, pu, su, pd, sd, H, F, x, idx, wts, np.arange(T))
    xv = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for t in range(T):
        acc = np.zeros(H)
        for j in range(K):
            e = idx[t, j]
            g = _decode(pg[e], sg[e], H, 64) @ xv[t]
            u = _decode(pu[e], su[e], H, 64) @ xv[t]
            h = g / (1 + np.exp(-g)) * u
            hb = np.array([oracle.round_bf16(v) for v in h])  # RNE to bf16 (pinned in test_oracle.py)
            acc += wts[t, j] * (_decode(pd[e], sd[e], F, 64) @ hb)
        # h summed in another order may round to bf16 one ulp apart on a rare element
        assert np.all(np.abs(y[t] - acc) <= 1e-4 * bound[t] + 1e-300)
