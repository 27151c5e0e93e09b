"""GPU parity of the next rows: quantisation (bit-exact codes and scales), row
dequantisation / gather, the matvec over selected rows, and the general group sizes of
gq4_matvec / gq4_gate_up_silu -- each against the CPU oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import (bf16_to_torch, check_bf16_close, check_close, device_words_to_host, h_bound,
                           torch_bf16_to_bits)
from weight_only_int4_gq4_b200 import synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from weight_only_int4_gq4_b200 import gq4


def _weights(seed, O, I, scale=1.0):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((O, I)) * rng.uniform(0.05, 2.0, size=(O, 1)) * scale).astype(np.float32)
    return w


def _host_bytes(T):
    """Packed bytes of a gq4 Tensor in the pages' low-nibble-first order."""
    O, I = T.out, T.in_
    return device_words_to_host(T.w.cpu().numpy().reshape(O, I // 2))


# ---------------------------------------------------------------- quantisation
@pytest.mark.parametrize("O,I,gs", [(64, 256, 64), (33, 200, 64), (16, 512, 128), (20, 96, 48), (12, 384, 96),
                                    (10, 256, 256), (9, 1024, 512), (7, 120, 120), (40, 64, 16), (8, 264, 8)])
def test_quantize_bitexact(O, I, gs):
    w = _weights(O * 7 + I, O, I)
    w[1, :gs] = 0.0  # an all-zero group
    w[2, 3] = 3.5 * w[2, :gs].__abs__().max() / 7  # a value near a rounding tie
    q_o, s_o = oracle.quantize(w, gs)
    T = gq4.quantize(torch.from_numpy(w).cuda(), gs)
    torch.cuda.synchronize()
    assert np.array_equal(T.s.cpu().numpy().reshape(s_o.shape), s_o)
    assert np.array_equal(_host_bytes(T), oracle.pack(q_o))


def test_quantize_full_expert_and_use():
    """A 6144 x 2048 expert matrix (the workloads' down projection), quantised on the GPU,
    bit-exact, then used by gq4_matvec against the oracle on the oracle's own codes."""
    O, I = 6144, 2048
    w = _weights(11, O, I, 0.02)
    q_o, s_o = oracle.quantize(w, 64)
    T = gq4.quantize(torch.from_numpy(w).cuda(), 64)
    torch.cuda.synchronize()
    assert np.array_equal(T.s.cpu().numpy().reshape(s_o.shape), s_o)
    assert np.array_equal(_host_bytes(T), oracle.pack(q_o))
    x = synth.x_normal(12, 2, I, "bf16", O, I, 2)
    y = gq4.matvec(T, bf16_to_torch(x)).cpu().numpy()
    rows = np.random.default_rng(13).choice(O, 64, replace=False)
    y_o, b = oracle.matvec(oracle.pack(q_o)[rows], s_o[rows], x)
    check_close(y[:, rows], y_o, b, "quantised expert matvec")


# ---------------------------------------------------------------- row dequantisation
def _packed(seed, O, I, gs):
    q = synth.q_uniform(seed, O, I, O, I, gs)
    s = synth.scales_uniform(seed, O, -(-I // gs), -0.02, 0.02, O, I, gs)
    return q, oracle.pack(q), s


@pytest.mark.parametrize("O,I,gs", [(100, 256, 64), (37, 200, 64), (50, 384, 96), (20, 4096, 128), (16, 72, 8)])
def test_dequant_rows_f32_bf16_accumulate(O, I, gs):
    q, p, s = _packed(O + I, O, I, gs)
    W = gq4.upload(p, s, gs=gs)
    rng = np.random.default_rng(gs)
    idx = rng.integers(0, O, size=9).astype(np.int32)
    idx_t = torch.from_numpy(idx).cuda()
    ref = oracle.dequant_rows(p, s, I, idx, gs)
    # f32: one rounding of s*q
    got = gq4.dequant_rows(W, idx_t).cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= 2.0 ** -24 * np.abs(ref))
    # bf16: the GPU rounds its f32 value, the oracle the exact value
    gb = torch_bf16_to_bits(gq4.dequant_rows(W, idx_t, dtype=torch.bfloat16))
    check_bf16_close(gb, np.vectorize(oracle.round_bf16)(ref), np.zeros_like(ref), "dequant bf16")
    # accumulate with alpha (qt_addrow): three f32 roundings at most
    alpha = rng.standard_normal(9).astype(np.float32)
    base = rng.standard_normal((9, I)).astype(np.float32)
    out = torch.from_numpy(base.copy()).cuda()
    gq4.dequant_rows(W, idx_t, alpha=torch.from_numpy(alpha).cuda(), out=out, accumulate=True)
    ref2 = oracle.dequant_rows(p, s, I, idx, gs, alpha=alpha.astype(np.float64), out=base.astype(np.float64))
    err = np.abs(out.cpu().numpy().astype(np.float64) - ref2)
    lim = 4 * 2.0 ** -24 * (np.abs(base) + np.abs(alpha[:, None].astype(np.float64) * ref) + np.abs(ref2))
    assert np.all(err <= lim)


def test_dequant_rows_out_of_range_index_gives_nan():
    q, p, s = _packed(3, 16, 128, 64)
    W = gq4.upload(p, s)
    idx = torch.tensor([0, 16, -1, 5], dtype=torch.int32, device="cuda")
    out = gq4.dequant_rows(W, idx).cpu().numpy()
    assert np.all(np.isnan(out[1])) and np.all(np.isnan(out[2]))
    assert np.all(np.isfinite(out[0])) and np.all(np.isfinite(out[3]))


# ---------------------------------------------------------------- matvec over rows
@pytest.mark.parametrize("O,I,gs,T,dt", [(300, 4096, 64, 1, "bf16"), (128, 200, 64, 3, "f32"), (64, 384, 96, 9, "bf16"),
                                         (2000, 1024, 128, 2, "bf16"), (40, 1536, 32, 5, "f32")])
def test_matvec_rows(O, I, gs, T, dt):
    q, p, s = _packed(O * 3 + I, O, I, gs)
    W = gq4.upload(p, s, gs=gs)
    idx = np.random.default_rng(T).integers(0, O, size=77).astype(np.int32)
    x = synth.x_normal(5, T, I, dt, O, I, T)
    xt = bf16_to_torch(x) if dt == "bf16" else torch.from_numpy(x).cuda()
    y = gq4.matvec_rows(W, torch.from_numpy(idx).cuda(), xt).cpu().numpy()
    y_o, b = oracle.matvec_rows(p, s, idx, x, gs)
    check_close(y, y_o, b, f"matvec_rows {O}x{I} gs={gs}")


def test_matvec_rows_vocab_sized():
    """Selected rows of an LM-head-sized matrix (151936 x 4096, gs = 64)."""
    O, I = 151936, 4096
    rng = np.random.default_rng(29)
    p = rng.integers(0, 256, size=(O, I // 2), dtype=np.uint8)
    s = rng.uniform(0.002, 0.02, size=(O, I // 64)).astype(np.float32)
    W = gq4.upload(p, s)
    idx = rng.integers(0, O, size=512).astype(np.int32)
    x = synth.x_normal(30, 1, I, "bf16", O, I, 1)
    y = gq4.matvec_rows(W, torch.from_numpy(idx).cuda(), bf16_to_torch(x)).cpu().numpy()
    y_o, b = oracle.matvec_rows(p, s, idx[:64], x)
    check_close(y[:, :64], y_o, b, "vocab rows")


# ---------------------------------------------------------------- general group sizes
@pytest.mark.parametrize("O,I,gs,T,dt", [(96, 256, 16, 1, "bf16"), (70, 512, 32, 4, "bf16"), (50, 480, 48, 2, "f32"),
                                         (130, 1024, 128, 3, "bf16"), (33, 200, 64, 1, "bf16"), (64, 1000, 64, 10, "f32"),
                                         (16, 4096, 256, 1, "bf16")])
def test_matvec_general_group_size(O, I, gs, T, dt):
    q, p, s = _packed(O + I + gs, O, I, gs)
    W = gq4.upload(p, s, gs=gs)
    x = synth.x_normal(9, T, I, dt, O, I, T)
    xt = bf16_to_torch(x) if dt == "bf16" else torch.from_numpy(x).cuda()
    y = gq4.matvec(W, xt).cpu().numpy()
    y_o, b = oracle.matvec(p, s, x, gs)
    check_close(y, y_o, b, f"matvec gs={gs} {O}x{I}")


@pytest.mark.parametrize("F,H,gs,T", [(64, 256, 32, 2), (48, 200, 64, 1), (40, 768, 128, 3)])
def test_gate_up_general_group_size(F, H, gs, T):
    qg, pg, sg = _packed(F + 1, F, H, gs)
    qu, pu, su = _packed(F + 2, F, H, gs)
    Wg, Wu = gq4.upload(pg, sg, gs=gs), gq4.upload(pu, su, gs=gs)
    x = synth.x_normal(4, T, H, "bf16", F, H, T)
    h = torch_bf16_to_bits(gq4.gate_up_silu(Wg, Wu, bf16_to_torch(x)))
    h_o, g_o, u_o = oracle.gate_up_silu(pg, sg, pu, su, x, gs)
    xmax = np.abs(synth.bf16_bits_to_f32(x)).max(1).astype(np.float64)
    b = h_bound(oracle.row_l1(pg, sg, H, gs), oracle.row_l1(pu, su, H, gs), xmax, g_o, u_o)
    check_bf16_close(h, h_o, b, f"gate_up gs={gs}")


@pytest.mark.parametrize("gs,I", [(64, 256), (32, 256), (128, 512)])
def test_matvec_rows_out_of_range_index_gives_nan(gs, I):
    q, p, s = _packed(gs + I, 40, I, gs)
    W = gq4.upload(p, s, gs=gs)
    idx = np.array([0, 40, 7, -3, 39], np.int32)
    x = synth.x_normal(2, 2, I, "bf16", 40, I, 2)
    y = gq4.matvec_rows(W, torch.from_numpy(idx).cuda(), bf16_to_torch(x)).cpu().numpy()
    assert np.all(np.isnan(y[:, 1])) and np.all(np.isnan(y[:, 3]))
    ok = [0, 2, 4]
    y_o, b = oracle.matvec_rows(p, s, idx[ok], x, gs)
    check_close(y[:, ok], y_o, b, f"matvec_rows valid columns gs={gs}")


# ---------------------------------------------------------------- MLA absorb projections
def _kvb(seed, nh, dn, dv, R, gs):
    O = nh * (dn + dv)
    packed = synth.packed_uniform(seed, O, R, 3)
    scales = synth.scales_uniform(seed, O, -(-R // gs), 0.002, 0.02, 3)
    return packed, scales


def _act(seed, shape, dt):
    x = synth.rng(seed, 5).standard_normal(shape).astype(np.float32)
    if dt == "bf16":
        xb = synth.to_bf16_bits(x)
        return xb, bf16_to_torch(xb)
    return x, torch.from_numpy(x).cuda()


@pytest.mark.parametrize("nh,dn,dv,R,gs,T,dt", [
    (64, 192, 256, 512, 64, 1, "bf16"),   # the pages' kv_b: 28,672 rows x 512, 8 groups per row
    (64, 192, 256, 512, 64, 5, "f32"),    # two token blocks, the second ragged
    (3, 5, 7, 40, 16, 6, "f32"),          # partial last group (40 = 16 + 16 + 8)
    (2, 9, 33, 24, 16, 3, "bf16"),        # value rows spill into a second block row range
    (4, 16, 8, 1024, 128, 2, "bf16"),     # 128 words per row: two key-row splits
    (2, 12, 20, 2048, 64, 4, "f32"),      # 256 words per row: one thread per word
    (1, 1, 1, 8, 8, 1, "f32"),            # one word, one group
])
def test_mla_absorb_q_and_v(nh, dn, dv, R, gs, T, dt):
    packed, scales = _kvb(nh * 1000 + R + gs, nh, dn, dv, R, gs)
    W = gq4.upload(packed, scales, gs=gs)
    qn_h, qn = _act(R + T, (T, nh, dn), dt)
    lat_h, lat = _act(R + T + 1, (T, nh, R), dt)
    q_lat = gq4.mla_absorb_q(W, nh, dn, dv, qn)
    o = gq4.mla_absorb_v(W, nh, dn, dv, lat)
    torch.cuda.synchronize()
    ref_q, b_q = oracle.mla_absorb_q(packed, scales, R, nh, dn, dv, qn_h, gs)
    ref_v, b_v = oracle.mla_absorb_v(packed, scales, R, nh, dn, dv, lat_h, gs)
    check_close(q_lat.cpu().numpy(), ref_q, b_q, "mla absorb q")
    check_close(o.cpu().numpy(), ref_v, b_v, "mla absorb v")
