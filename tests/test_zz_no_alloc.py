"""moe_expert_ffn_noalloc: the MoE layer for callers that cannot allocate device memory.

Some hosts own every device allocation themselves (a plug-in receives only the tensors it
works on), and some decode loops must not call cudaMalloc because it can synchronise the
device.  For them the library keeps one fixed-size device array per GPU and uses it in
place of the caller's workspace.  These tests check that this entry point, called through
the C ABI, gives the oracle's results and those of the workspace entry point on two
calls in a row (the second one after the first has left its contents in the shared
array), and that a shape too large for the array is refused before anything is
launched.

This file is named to be collected last: if it fails, a run that stops at the first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from weight_only_int4_gq4_b200 import gq4, synth
from tests.helpers import bf16_to_torch, check_close


def _stacked(cfg):
    parts = {n: [getattr(cfg, n)(e) for e in range(cfg.E)] for n in ("gate", "up", "down")}
    return {n: (np.stack([a for a, _ in v]), np.stack([b for _, b in v])) for n, v in parts.items()}


def _noalloc(W, lg, x, K, y, status):
    """One call of the C entry point (argument marshalling only)."""
    T, H = x.shape
    E = lg.shape[1]
    return gq4.lib().moe_expert_ffn_noalloc(
        W["gate"].ref(), W["up"].ref(), W["down"].ref(), ctypes.c_void_p(lg.data_ptr()),
        ctypes.c_void_p(x.data_ptr()), gq4.BF16, T, E, K, ctypes.c_void_p(y.data_ptr()),
        ctypes.c_void_p(status.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_two_calls():
    torch.cuda.set_device(0)
    # first call: few rows per expert (decode kernels); second call: experts with more
    # than 32 rows on shapes the tensor-core kernels take (H and F multiples of 256), so
    # the row gather and the tensor-core kernels run through the array as well
    cases = [synth.MoEConfig("noalloc_t6_e8_k2", T=6, H=256, E=8, F=128, K=2, seed=41),
             synth.MoEConfig("noalloc_t80_e4_k2", T=80, H=256, E=4, F=256, K=2, seed=42)]
    for i, cfg in enumerate(cases):
        st = _stacked(cfg)
        W = {n: gq4.upload(*st[n]) for n in st}
        lg_h, _ = cfg.logits()
        x_h = cfg.x()
        lg = torch.from_numpy(lg_h).cuda()
        x = bf16_to_torch(x_h)
        y_ref, ws = gq4.moe_expert_ffn(W["gate"], W["up"], W["down"], lg, x, cfg.K)
        assert ws.status() == 0
        if i == 1:  # the second call reaches the tensor-core kernels
            assert int(ws.routing()["cnt"].max()) >= gq4.MOE_LARGE_MIN_ROWS
        y = torch.full((cfg.T, cfg.H), float("nan"), dtype=torch.float32, device="cuda")
        status = torch.full((4,), -1, dtype=torch.int32, device="cuda")
        assert _noalloc(W, lg, x, cfg.K, y, status) == gq4.OK
        torch.cuda.synchronize()
        assert int(status[0]) == 0
        _, idx, wts, _ = oracle.route(lg_h, cfg.K)
        y_o, bound = oracle.moe_tokens(*st["gate"], *st["up"], *st["down"], cfg.H, cfg.F, x_h, idx, wts,
                                       np.arange(cfg.T))
        # against the oracle, and against the workspace entry point
        check_close(y.cpu().numpy(), y_o, bound, cfg.name + " vs oracle")
        check_close(y.cpu().numpy(), y_ref.cpu().numpy(), bound, cfg.name + " vs moe_expert_ffn")


def test_noalloc_rejects_shapes_beyond_the_array():
    """A shape whose workspace exceeds the array is refused on the host (no GPU needed:
    the size check comes before any CUDA call, so the fake pointers are never used)."""
    T, E, K, H, F = 4096, 256, 8, 6144, 2048
    assert gq4.moe_workspace_bytes(T, E, K, H, F) > gq4.NOALLOC_SCRATCH_BYTES
    fake = 1 << 40
    desc = {}
    for name, (O, I) in (("gate", (F, H)), ("up", (F, H)), ("down", (H, F))):
        d = gq4.TensorDesc()
        assert gq4.lib().gq4_tensor_init(fake, fake, O, I, 64, E, ctypes.byref(d)) == gq4.OK
        desc[name] = d
    st = gq4.lib().moe_expert_ffn_noalloc(
        ctypes.byref(desc["gate"]), ctypes.byref(desc["up"]), ctypes.byref(desc["down"]), fake, fake,
        gq4.BF16, T, E, K, fake, None, None)
    assert st == gq4.ERR_WORKSPACE


def test_noalloc_rejects_a_status_word_inside_a_weight_buffer():
    """The status word is copied after the layer, so it may not lie inside any input:
    one placed inside a weight or scale array is refused on the host before any CUDA
    call (fake, never dereferenced device addresses)."""
    T, E, K, H, F = 4, 4, 2, 256, 256
    base = 1 << 40
    desc = {}
    for i, (name, (O, I)) in enumerate((("gate", (F, H)), ("up", (F, H)), ("down", (H, F)))):
        d = gq4.TensorDesc()
        w, s = base + i * (1 << 30), base + i * (1 << 30) + (1 << 28)
        assert gq4.lib().gq4_tensor_init(w, s, O, I, 64, E, ctypes.byref(d)) == gq4.OK
        desc[name] = d
    io = base + (8 << 30)
    for status_at in (desc["down"].w + 4096, desc["up"].s + 64, desc["gate"].w):
        st = gq4.lib().moe_expert_ffn_noalloc(
            ctypes.byref(desc["gate"]), ctypes.byref(desc["up"]), ctypes.byref(desc["down"]), io,
            io + (1 << 20), gq4.BF16, T, E, K, io + (2 << 20), status_at, None)
        assert st == gq4.ERR_ALIAS, hex(status_at)
