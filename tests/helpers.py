"""Shared helpers of the GPU parity tests: tolerance checks and input marshalling."""
from __future__ import annotations

import numpy as np
import torch

from weight_only_int4_gq4_b200 import synth

# Acceptance of the method statement: per element |err| <= 2e-3 * B (B = the sum of
# |terms| scale, "compare against the sum of |terms|"), relative L2 <= 1e-4.
ELEM_TOL = 2e-3
REL_L2_TOL = 1e-4
# bf16-valued outputs (h): the GPU rounds its f32 value, the oracle its fp64 value, so
# the two may straddle a rounding boundary; allowed: at most this fraction of elements
# one bf16 ulp apart (plus the per-element bound), all others equal.
BF16_FLIP_FRAC = 5e-3


def bf16_to_torch(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16).to(device)


def torch_bf16_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def device_words_to_host(dev: np.ndarray) -> np.ndarray:
    """Undo the device nibble order (even-k nibbles in the low half-word, odd-k in the
    high half-word of each 32-bit word) to get the pages' low-nibble-first bytes."""
    w = dev.reshape(dev.shape[0], -1).view(np.uint32)
    nib = np.stack([(w >> (4 * i)) & 15 for i in range(8)], -1)  # slots 0..7
    k = np.empty_like(nib)
    k[..., 0::2] = nib[..., 0:4]
    k[..., 1::2] = nib[..., 4:8]
    host = np.zeros_like(w)
    for i in range(8):
        host |= (k[..., i] << (4 * i)).astype(np.uint32)
    return host.view(np.uint8).reshape(dev.shape)


def check_close(y_gpu, y_orc, bound, what=""):
    y_gpu = np.asarray(y_gpu, np.float64)
    y_orc = np.asarray(y_orc, np.float64)
    assert y_gpu.shape == y_orc.shape, what
    assert np.all(np.isfinite(y_gpu)), what
    err = np.abs(y_gpu - y_orc)
    lim = ELEM_TOL * np.asarray(bound, np.float64)
    bad = err > lim
    assert not bad.any(), f"{what}: {bad.sum()} elements over 2e-3*B, worst ratio {(err / np.maximum(lim, 1e-300)).max():.3g}"
    denom = np.linalg.norm(y_orc)
    rel = np.linalg.norm(y_gpu - y_orc) / denom if denom > 0 else np.linalg.norm(y_gpu)
    assert rel <= REL_L2_TOL, f"{what}: relative L2 {rel:.3g}"
    return rel


def bf16_ulp(v):
    v = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(v, 2.0 ** -126)))
    return np.ldexp(1.0, (e - 7).astype(np.int64))


def check_bf16_close(h_gpu_bits, h_orc, bound, what=""):
    """h_gpu as bf16 bits, h_orc as fp64 values already rounded to bf16."""
    h_gpu = synth.bf16_bits_to_f32(h_gpu_bits).astype(np.float64)
    h_orc = np.asarray(h_orc, np.float64)
    assert np.all(np.isfinite(h_gpu)), what
    diff = h_gpu != h_orc
    frac = diff.mean()
    assert frac <= BF16_FLIP_FRAC, f"{what}: {diff.sum()} of {diff.size} differ"
    err = np.abs(h_gpu - h_orc)
    lim = bf16_ulp(h_orc) * 1.0000001 + ELEM_TOL * np.asarray(bound, np.float64)
    assert np.all(err <= lim), f"{what}: worst {(err / lim).max():.3g}"
    return frac


def h_bound(l1g, l1u, xmax, g, u):
    """Per-element scale of an h = silu(g)*u error: |dsilu/dg| <= 1.1 times the gate's
    sum-of-|terms| scale times |u|, plus |silu(g)| times the up scale."""
    silu = g / (1 + np.exp(-g))
    return 1.1 * l1g[None, :] * xmax[:, None] * np.abs(u) + np.abs(silu) * l1u[None, :] * xmax[:, None]
