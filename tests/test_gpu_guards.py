"""Failure detection without a GPU fault.

* Guard bands: each output is a window inside a larger buffer whose margins hold a
  sentinel bit pattern; after the call the margins must be untouched, so a kernel that
  writes past its output (a ragged tail, a partial tile) fails here instead of corrupting
  a neighbour.  Shapes are ragged on purpose (row counts not multiples of the tiles).
* Bounded waits: every wait of the library's kernels gives up after a time limit and
  reports GQ4_ERR_TIMEOUT in the status word.  gq4_selftest_wait_timeout runs that wait on
  a barrier nothing completes, with a 1 ms limit: the status must say timeout and the
  context must stay usable (a matvec afterwards still matches the oracle).
"""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import bf16_to_torch, check_close
from weight_only_int4_gq4_b200 import synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from weight_only_int4_gq4_b200 import gq4

SENTINEL = 0x7FC0DEAD  # a NaN payload no kernel writes
GUARD = 1024           # 32-bit words of margin on each side (16-byte aligned window)


def guarded(shape, dtype=torch.float32):
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    words = (n + 3) // 4
    buf = torch.full((words + 2 * GUARD,), SENTINEL, dtype=torch.int32, device="cuda")
    win = buf[GUARD:GUARD + words].view(torch.uint8)[:n].view(dtype).view(shape)
    return buf, win


def intact(buf, words):
    torch.cuda.synchronize()
    b = buf.cpu().numpy()
    return np.all(b[:GUARD] == SENTINEL) and np.all(b[GUARD + words:] == SENTINEL)


def _words(t):
    return (t.numel() * t.element_size() + 3) // 4


def _tensor(seed, O, I, gs=64):
    p = synth.packed_uniform(seed, O, I, 7)
    s = synth.scales_uniform(seed, O, -(-I // gs), 0.002, 0.02, 7)
    return p, s, gq4.upload(p, s, gs=gs)


@pytest.mark.parametrize("O,I,T,gs", [(200, 512, 1, 64), (333, 1024, 5, 64), (70, 256, 2, 32), (1000, 4096, 3, 64)])
def test_matvec_and_gate_up_stay_in_bounds(O, I, T, gs):
    p, s, W = _tensor(O + I, O, I, gs)
    _, _, W2 = _tensor(O + I + 1, O, I, gs)
    x = bf16_to_torch(synth.x_normal(3, T, I, "bf16"))
    buf, y = guarded((T, O))
    gq4.matvec(W, x, y)
    assert intact(buf, _words(y))
    y_o, b = oracle.matvec(p, s, synth.x_normal(3, T, I, "bf16"), gs)
    check_close(y.cpu().numpy(), y_o, b, "guarded matvec")
    buf, h = guarded((T, O), torch.bfloat16)
    gq4.gate_up_silu(W, W2, x, h)
    assert intact(buf, _words(h))


@pytest.mark.parametrize("T,E,K,H,F", [(5, 4, 2, 256, 192), (40, 8, 4, 384, 192), (70, 3, 2, 128, 64),
                                       # tensor-core kernels: 45 rows per expert (not a multiple
                                       # of 16), and 60-80 rows beside decode-path experts
                                       (45, 2, 2, 256, 256), (100, 5, 2, 512, 256)])
def test_moe_output_stays_in_bounds(T, E, K, H, F):
    cfg = synth.MoEConfig(f"guard_t{T}_e{E}", T=T, H=H, E=E, F=F, K=K, seed=T + E)
    parts = {n: [getattr(cfg, n)(e) for e in range(E)] for n in ("gate", "up", "down")}
    W = {n: gq4.upload(np.stack([a for a, _ in v]), np.stack([b for _, b in v])) for n, v in parts.items()}
    lg, _ = cfg.logits()
    buf, y = guarded((T, H))
    _, ws = gq4.moe_expert_ffn(W["gate"], W["up"], W["down"], torch.from_numpy(lg).cuda(),
                               bf16_to_torch(cfg.x()), K, y=y)
    assert ws.status() == 0
    assert intact(buf, _words(y))
    if H % 256 == 0 and F % 256 == 0 and T >= gq4.MOE_LARGE_MIN_ROWS:
        assert int(ws.routing()["cnt"].max()) >= gq4.MOE_LARGE_MIN_ROWS  # reaches the tensor cores


def test_row_ops_and_mla_stay_in_bounds():
    O, I = 301, 512
    p, s, W = _tensor(11, O, I)
    idx = torch.tensor([0, 300, 17, 5, 299], dtype=torch.int32, device="cuda")
    buf, out = guarded((5, I))
    gq4.dequant_rows(W, idx, out=out)
    assert intact(buf, _words(out))
    x = bf16_to_torch(synth.x_normal(4, 3, I, "bf16"))
    buf, y = guarded((3, 5))
    gq4.matvec_rows(W, idx, x, y)
    assert intact(buf, _words(y))
    nh, dn, dv, R = 3, 7, 5, 136
    _, _, Wk = _tensor(12, nh * (dn + dv), R, 8)
    qn = torch.randn(6, nh, dn, device="cuda")
    lat = torch.randn(6, nh, R, device="cuda")
    buf, ql = guarded((6, nh, R))
    gq4.mla_absorb_q(Wk, nh, dn, dv, qn, ql)
    assert intact(buf, _words(ql))
    buf, o = guarded((6, nh, dv))
    gq4.mla_absorb_v(Wk, nh, dn, dv, lat, o)
    assert intact(buf, _words(o))


def test_bounded_wait_gives_up_and_the_context_survives():
    torch.cuda.synchronize()
    assert gq4.selftest_wait_timeout(1000) == gq4.ERR_TIMEOUT
    # the context is still usable: a matvec after the timed-out wait matches the oracle
    p, s, W = _tensor(21, 96, 256)
    xh = synth.x_normal(5, 2, 256, "bf16")
    y = gq4.matvec(W, bf16_to_torch(xh)).cpu().numpy()
    y_o, b = oracle.matvec(p, s, xh)
    check_close(y, y_o, b, "matvec after the wait self-test")


def test_sync_status_reads_the_router_status_word():
    """A router row with a NaN logit raises GQ4_ERR_NONFINITE_LOGIT in the status word;
    gq4_sync_status waits for the stream and reads it."""
    lg = torch.randn(3, 16, device="cuda")
    lg[1, 4] = float("nan")
    _, _, st = gq4.route(lg, 2)
    assert gq4.sync_status(st) == gq4.ERR_NONFINITE_LOGIT
    _, _, st = gq4.route(torch.randn(3, 16, device="cuda"), 2)
    assert gq4.sync_status(st) == 0
