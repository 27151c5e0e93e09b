"""CPU oracle for the grouped-int4 (fmt=4, gs=64) MoE expert FFN.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package; the product library never does.

This module is argument marshalling around ``gq4_oracle.c`` (plain C, fp64), which
holds every step of the arithmetic.  It shares no code with the CUDA path.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gq4_oracle.c")
_LIB = os.path.join(_HERE, "_liboracle.so")

OK = 0
ERR_SHAPE = 3
ERR_NONFINITE_LOGIT = 9

F32 = 0
BF16 = 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP over independent outputs, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c99", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
            "-Wall", "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        L = _lib
        L.orc_nibble_to_q.argtypes = [I, I]
        L.orc_nibble_to_q.restype = I
        L.orc_unpack.argtypes = [P, I64, I64, I64, I]
        L.orc_unpack.restype = I
        L.orc_pack.argtypes = [P, I64, I64, I, P]
        L.orc_pack.restype = None
        L.orc_ngroups.argtypes = [I64, I64]
        L.orc_ngroups.restype = I64
        L.orc_weight_bytes.argtypes = [I64, I64]
        L.orc_weight_bytes.restype = I64
        L.orc_scale_bytes.argtypes = [I64, I64, I64]
        L.orc_scale_bytes.restype = I64
        L.orc_weight.argtypes = [P, P, I64, I64, I64, I64, I64]
        L.orc_weight.restype = ctypes.c_double
        L.orc_matvec.argtypes = [P, P, I64, I64, I64, P, I, I64, P, P]
        L.orc_matvec.restype = None
        L.orc_row_l1.argtypes = [P, P, I64, I64, I64, P]
        L.orc_row_l1.restype = None
        L.orc_round_bf16.argtypes = [ctypes.c_double]
        L.orc_round_bf16.restype = ctypes.c_double
        L.orc_gate_up_silu.argtypes = [P, P, P, P, I64, I64, I64, P, I, I64, I, P, P, P]
        L.orc_gate_up_silu.restype = None
        L.orc_route.argtypes = [P, I64, I64, I64, P, P, P]
        L.orc_route.restype = I
        L.orc_rowmap.argtypes = [P, I64, I64, I64, P, P, P, P, P]
        L.orc_rowmap.restype = I
        L.orc_moe_tokens.argtypes = [P, P, P, P, P, P, I64, I64, I64, I64, I64, I64, I64,
                                     P, I, I, P, P, I64, P, I64, P, P]
        L.orc_moe_tokens.restype = None
        L.orc_detect_group_size.argtypes = [I64, I64, I64]
        L.orc_detect_group_size.restype = I64
        L.orc_quantize.argtypes = [P, I64, I64, I64, P, P]
        L.orc_quantize.restype = None
        L.orc_dequant_rows.argtypes = [P, P, I64, I64, I64, P, I64, P, I, P]
        L.orc_dequant_rows.restype = None
        L.orc_matvec_rows.argtypes = [P, P, I64, I64, I64, P, I64, P, I, I64, P, P]
        L.orc_mla_absorb_q.argtypes = [P, P, I64, I64, I64, I64, I64, P, I, I64, P, P]
        L.orc_mla_absorb_q.restype = None
        L.orc_mla_absorb_v.argtypes = [P, P, I64, I64, I64, I64, I64, P, I, I64, P, P]
        L.orc_mla_absorb_v.restype = None
        L.orc_set_threads.argtypes = [I]
        L.orc_set_threads.restype = I
        L.orc_matvec_rows.restype = None
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _xdt(x: np.ndarray) -> int:
    if x.dtype == np.float32:
        return F32
    if x.dtype == np.uint16:  # bf16 bit patterns
        return BF16
    raise TypeError("x must be float32 or uint16 (bf16 bits)")


def nibble_to_q(nibble: int, offset_binary: bool = False) -> int:
    return lib().orc_nibble_to_q(int(nibble), int(offset_binary))


def pack(q: np.ndarray, offset_binary: bool = False) -> np.ndarray:
    """q int8 [O][I] in -8..7 -> packed uint8 [O][(I+1)//2]."""
    q = _c(q, np.int8)
    O, I = q.shape
    out = np.empty((O, (I + 1) // 2), np.uint8)
    lib().orc_pack(_p(q), O, I, int(offset_binary), _p(out))
    return out


def unpack(packed: np.ndarray, I: int, offset_binary: bool = False) -> np.ndarray:
    packed = _c(packed, np.uint8)
    O = packed.shape[0]
    rb = packed.shape[1]
    L = lib()
    out = np.empty((O, I), np.int8)
    for o in range(O):
        for k in range(I):
            out[o, k] = L.orc_unpack(_p(packed), rb, o, k, int(offset_binary))
    return out


def ngroups(I: int, gs: int) -> int:
    return lib().orc_ngroups(I, gs)


def weight_bytes(O: int, I: int) -> int:
    return lib().orc_weight_bytes(O, I)


def scale_bytes(O: int, I: int, gs: int) -> int:
    return lib().orc_scale_bytes(O, I, gs)


def weight(packed, scales, I, gs, o, k) -> float:
    packed = _c(packed, np.uint8)
    scales = _c(scales, np.float32)
    return lib().orc_weight(_p(packed), _p(scales), packed.shape[0], I, gs, o, k)


def matvec(packed, scales, x, gs: int = 64):
    """y[t][o] in fp64 and the Sigma|terms| bound; x [T][I] f32 or bf16 bits."""
    packed = _c(packed, np.uint8)
    scales = _c(scales, np.float32)
    x = np.ascontiguousarray(x)
    if x.ndim == 1:
        x = x[None]
    T, I = x.shape
    O = packed.shape[0]
    y = np.empty((T, O), np.float64)
    b = np.empty((T, O), np.float64)
    lib().orc_matvec(_p(packed), _p(scales), O, I, gs, _p(x), _xdt(x), T, _p(y), _p(b))
    return y, b


def row_l1(packed, scales, I, gs: int = 64):
    packed = _c(packed, np.uint8)
    scales = _c(scales, np.float32)
    O = packed.shape[0]
    out = np.empty(O, np.float64)
    lib().orc_row_l1(_p(packed), _p(scales), O, I, gs, _p(out))
    return out


def round_bf16(v: float) -> float:
    return lib().orc_round_bf16(float(v))


def gate_up_silu(pg, sg, pu, su, x, gs: int = 64, hdt: int | None = None):
    """h [T][F] (fp64 values already rounded to hdt), plus g and u in fp64."""
    pg, pu = _c(pg, np.uint8), _c(pu, np.uint8)
    sg, su = _c(sg, np.float32), _c(su, np.float32)
    x = np.ascontiguousarray(x)
    if x.ndim == 1:
        x = x[None]
    T, H = x.shape
    F = pg.shape[0]
    xdt = _xdt(x)
    if hdt is None:
        hdt = xdt
    h = np.empty((T, F), np.float64)
    g = np.empty((T, F), np.float64)
    u = np.empty((T, F), np.float64)
    lib().orc_gate_up_silu(_p(pg), _p(sg), _p(pu), _p(su), F, H, gs, _p(x), xdt, T, hdt,
                           _p(h), _p(g), _p(u))
    return h, g, u


def route(logits, K: int):
    """-> (status, idx int32 [T][K], wts fp64 [T][K], bad int32 [T])."""
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, K), np.int32)
    wts = np.empty((T, K), np.float64)
    bad = np.empty(T, np.int32)
    st = lib().orc_route(_p(logits), T, E, K, _p(idx), _p(wts), _p(bad))
    return st, idx, wts, bad


def rowmap(idx, E: int):
    """-> dict of cnt [E], offs [E+1], row_tok, row_slot, slot_row [T*K] (int32)."""
    idx = _c(idx, np.int32)
    T, K = idx.shape
    n = T * K
    cnt = np.empty(E, np.int32)
    offs = np.empty(E + 1, np.int32)
    row_tok = np.empty(n, np.int32)
    row_slot = np.empty(n, np.int32)
    slot_row = np.empty(n, np.int32)
    st = lib().orc_rowmap(_p(idx), T, K, E, _p(cnt), _p(offs), _p(row_tok), _p(row_slot),
                          _p(slot_row))
    if st != OK:
        raise ValueError("rowmap: expert index out of range")
    return dict(cnt=cnt, offs=offs, row_tok=row_tok, row_slot=row_slot, slot_row=slot_row)


def moe_tokens(pg, sg, pu, su, pd, sd, H, F, x, idx, wts, tokens, gs: int = 64,
               hdt: int | None = None):
    """MoE output y [n][H] (fp64) and bound [n][H] for the listed tokens.

    pg/pu: uint8 [E][F][H/2]; sg/su: f32 [E][F][ng_H]; pd: uint8 [E][H][F/2];
    sd: f32 [E][H][ng_F]; x [T][H] f32 or bf16 bits; idx int32 [T][K]; wts fp64 [T][K].
    """
    pg, pu, pd = _c(pg, np.uint8), _c(pu, np.uint8), _c(pd, np.uint8)
    sg, su, sd = _c(sg, np.float32), _c(su, np.float32), _c(sd, np.float32)
    x = np.ascontiguousarray(x)
    idx = _c(idx, np.int32)
    wts = _c(wts, np.float64)
    tokens = _c(tokens, np.int64)
    K = idx.shape[1]
    xdt = _xdt(x)
    if hdt is None:
        hdt = xdt
    n = tokens.shape[0]
    y = np.empty((n, H), np.float64)
    b = np.empty((n, H), np.float64)
    E = pg.shape[0]
    wgu = pg[0].size if E else 0
    sgu = sg[0].size if E else 0
    wd = pd[0].size if E else 0
    sdd = sd[0].size if E else 0
    lib().orc_moe_tokens(_p(pg), _p(sg), _p(pu), _p(su), _p(pd), _p(sd), wgu, sgu, wd, sdd,
                         H, F, gs, _p(x), xdt, hdt, _p(idx), _p(wts), K, _p(tokens), n,
                         _p(y), _p(b))
    return y, b


# ------------------------------------------------------------------ NEXT rows
def detect_group_size(O: int, I: int, scale_bytes: int) -> int:
    """The one candidate group size matching the scale array's size; 0 none, -1 several."""
    return lib().orc_detect_group_size(O, I, scale_bytes)


def quantize(w, gs: int = 64):
    """w f32 [O][I] -> (q int8 [O][I], scales f32 [O][ceil(I/gs)])."""
    w = _c(w, np.float32)
    O, I = w.shape
    q = np.empty((O, I), np.int8)
    s = np.empty((O, ngroups(I, gs)), np.float32)
    lib().orc_quantize(_p(w), O, I, gs, _p(q), _p(s))
    return q, s


def dequant_rows(packed, scales, I, idx, gs: int = 64, alpha=None, out=None):
    """out [n][I] fp64: alpha_j * w(idx[j], :) (+ out when out is given)."""
    packed = _c(packed, np.uint8)
    scales = _c(scales, np.float32)
    idx = _c(idx, np.int32)
    n = idx.shape[0]
    acc = out is not None
    o = _c(out, np.float64).copy() if acc else np.empty((n, I), np.float64)
    a = None if alpha is None else _c(alpha, np.float64)
    lib().orc_dequant_rows(_p(packed), _p(scales), packed.shape[0], I, gs, _p(idx), n,
                           None if a is None else _p(a), int(acc), _p(o))
    return o


def matvec_rows(packed, scales, idx, x, gs: int = 64):
    """y [T][n] fp64 over the rows idx, and the Sigma|terms| bound."""
    packed = _c(packed, np.uint8)
    scales = _c(scales, np.float32)
    idx = _c(idx, np.int32)
    x = np.ascontiguousarray(x)
    if x.ndim == 1:
        x = x[None]
    T, I = x.shape
    n = idx.shape[0]
    y = np.empty((T, n), np.float64)
    b = np.empty((T, n), np.float64)
    lib().orc_matvec_rows(_p(packed), _p(scales), packed.shape[0], I, gs, _p(idx), n, _p(x),
                          _xdt(x), T, _p(y), _p(b))
    return y, b


def _mla(fn, packed, scales, R, nh, dn, dv, x, width, gs):
    packed = _c(packed, np.uint8)
    scales = _c(scales, np.float32)
    x = np.ascontiguousarray(x)
    assert packed.shape[0] == nh * (dn + dv) and x.shape[-2:] == (nh, width), (packed.shape, x.shape)
    T = x.shape[0]
    n_out = R if fn == "q" else dv
    y = np.empty((T, nh, n_out), np.float64)
    b = np.empty((T, nh, n_out), np.float64)
    f = lib().orc_mla_absorb_q if fn == "q" else lib().orc_mla_absorb_v
    f(_p(packed), _p(scales), R, gs, nh, dn, dv, _p(x), _xdt(x), T, _p(y), _p(b))
    return y, b


def mla_absorb_q(packed, scales, R, nh, dn, dv, q_nope, gs: int = 64):
    """q_lat [T][nh][R] fp64 = sum_d q_nope[t][h][d] * w(h*(dn+dv)+d, c), and its bound.
    q_nope [T][nh][dn] f32 or bf16 bits (uint16)."""
    return _mla("q", packed, scales, R, nh, dn, dv, q_nope, dn, gs)


def mla_absorb_v(packed, scales, R, nh, dn, dv, lat, gs: int = 64):
    """o [T][nh][dv] fp64 = sum_c lat[t][h][c] * w(h*(dn+dv)+dn+v, c), and its bound.
    lat [T][nh][R] f32 or bf16 bits (uint16)."""
    return _mla("v", packed, scales, R, nh, dn, dv, lat, R, gs)


def set_threads(n: int) -> int:
    """Threads of the oracle's OpenMP loops; returns the previous count."""
    return lib().orc_set_threads(int(n))
