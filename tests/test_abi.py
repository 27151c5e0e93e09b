"""Host-side tests of the C ABI (no GPU needed): the library loads, exports every call
include/gq4.h declares, the host packer matches the oracle's, and every argument check
rejects bad input before anything is launched (fake device pointers are never touched
because validation fails first)."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from weight_only_int4_gq4_b200 import gq4, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "gq4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b((?:gq4|moe)_\w+)\s*\(", src)))


def test_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 15
    lib = gq4.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(gq4.EXPORTED)


def test_abi_version_and_status_strings():
    lib = gq4.lib()
    assert lib.gq4_abi_version() == 7
    for st in range(10):
        assert lib.gq4_status_string(st).decode()
    assert lib.gq4_status_string(77) == b"unknown status"


@pytest.mark.parametrize("O,I", [(1, 1), (4, 7), (16, 64), (3, 1000)])
def test_pack_matches_oracle(O, I):
    q = synth.q_uniform(12, O, I, O, I)
    assert np.array_equal(gq4.pack(q), oracle.pack(q))
    u = (q.astype(np.int16) + 8).astype(np.int8)  # offset-binary input nibbles
    assert np.array_equal(gq4.pack(u, offset_binary=True), oracle.pack(q))


def test_pack_rejects_out_of_range():
    with pytest.raises(gq4.GQ4Error) as e:
        gq4.pack(np.array([[8, 0]], np.int8))
    assert e.value.status == gq4.ERR_SHAPE
    with pytest.raises(gq4.GQ4Error):
        gq4.pack(np.array([[16, 0]], np.int8), offset_binary=True)


def test_device_bytes_worked_examples():
    assert gq4.device_bytes(28672, 512) == (7340032, 917504)  # kv_b
    w, s = gq4.device_bytes(2048, 6144, 64, 256)
    assert w == 256 * 6291456 and s == 256 * 786432


def _desc(out=64, in_=128, gs=64, w=0x10000, s=0x20000, E=1):
    d = gq4.TensorDesc()
    d.out, d.in_, d.gs, d.ng, d.n_experts = out, in_, gs, -(-in_ // gs), E
    d.w, d.s = w, s
    d.expert_stride_w, d.expert_stride_s = out * ((in_ + 1) // 2), out * d.ng
    return d


def _matvec(d, x=0x30000, y=0x40000, xdt=1, T=1):
    return gq4.lib().gq4_matvec(ctypes.byref(d), x, xdt, T, y, None)


def test_matvec_argument_checks():
    assert _matvec(_desc(w=0)) == gq4.ERR_NULL
    assert _matvec(_desc(), x=0) == gq4.ERR_NULL
    assert _matvec(_desc(w=0x10008)) == gq4.ERR_ALIGN
    assert _matvec(_desc(), y=0x40004) == gq4.ERR_ALIGN
    assert _matvec(_desc(gs=12)) == gq4.ERR_UNSUPPORTED          # gs not a multiple of 8
    assert _matvec(_desc(in_=100)) == gq4.ERR_UNSUPPORTED        # in not a multiple of 8
    bad = _desc()
    bad.ng = 3
    assert _matvec(bad) == gq4.ERR_SHAPE                          # ng inconsistent with in
    assert _matvec(_desc(), T=0) == gq4.ERR_SHAPE
    assert _matvec(_desc(), xdt=5) == gq4.ERR_UNSUPPORTED
    # y overlapping x or the weights
    assert _matvec(_desc(), x=0x40000, y=0x40000) == gq4.ERR_ALIAS
    assert _matvec(_desc(w=0x10000), y=0x10000) == gq4.ERR_ALIAS


def test_gate_up_argument_checks():
    L = gq4.lib()
    g, u = _desc(), _desc(w=0x50000, s=0x60000)
    u2 = _desc(out=32, w=0x50000, s=0x60000)
    assert L.gq4_gate_up_silu(ctypes.byref(g), ctypes.byref(u2), 0x30000, 1, 1, 0x70000, None) == gq4.ERR_SHAPE
    assert L.gq4_gate_up_silu(ctypes.byref(g), ctypes.byref(u), 0x30000, 1, 1, 0x30000, None) == gq4.ERR_ALIAS
    assert L.gq4_gate_up_silu(ctypes.byref(g), ctypes.byref(u), 0x30000, 1, 1, 0, None) == gq4.ERR_NULL


def test_route_rowmap_argument_checks():
    L = gq4.lib()
    assert L.gq4_route(0x1000, 4, 8, 9, 0x2000, 0x3000, 0x4000, None) == gq4.ERR_SHAPE  # K > E
    assert L.gq4_route(0x1000, 4, 2000, 8, 0x2000, 0x3000, 0x4000, None) == gq4.ERR_SHAPE  # E > 1024
    assert L.gq4_route(0x1000, 4, 8, 2, 0x1000, 0x3000, 0x4000, None) == gq4.ERR_ALIAS
    assert L.gq4_route(0x1004, 4, 8, 2, 0x2000, 0x3000, 0x4000, None) == gq4.ERR_ALIGN
    sb = L.gq4_rowmap_scratch_bytes(4, 2, 8)
    assert sb > 0
    args = [0x1000, 4, 2, 8, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 0x7000, 0x8000, 0x9000]
    assert L.gq4_rowmap(*args, sb - 1, None) == gq4.ERR_WORKSPACE
    args2 = list(args)
    args2[4] = 0x1000  # cnt overlaps idx
    assert L.gq4_rowmap(*args2, sb, None) == gq4.ERR_ALIAS


def test_moe_argument_checks():
    L = gq4.lib()
    T, E, K, H, F = 4, 8, 2, 128, 64
    wg = _desc(out=F, in_=H, w=0x100000, s=0x200000, E=E)
    wu = _desc(out=F, in_=H, w=0x300000, s=0x400000, E=E)
    wd = _desc(out=H, in_=F, w=0x500000, s=0x600000, E=E)
    ws_bytes = L.moe_expert_ffn_workspace_bytes(T, E, K, H, F)
    assert ws_bytes > T * K * F * 2

    def call(**kw):
        a = dict(g=wg, u=wu, d=wd, logits=0x700000, x=0x710000, xdt=1, T=T, E=E, K=K, y=0x720000,
                 ws=0x800000, wsb=ws_bytes)
        a.update(kw)
        return L.moe_expert_ffn(ctypes.byref(a["g"]), ctypes.byref(a["u"]), ctypes.byref(a["d"]),
                                a["logits"], a["x"], a["xdt"], a["T"], a["E"], a["K"], a["y"], a["ws"],
                                a["wsb"], None, None)

    assert call(wsb=ws_bytes - 1) == gq4.ERR_WORKSPACE
    assert call(xdt=0) == gq4.ERR_UNSUPPORTED
    assert call(K=9) == gq4.ERR_SHAPE
    assert call(d=_desc(out=H, in_=F, w=0x500000, s=0x600000, E=4)) == gq4.ERR_SHAPE  # too few experts
    assert call(y=0x710000) == gq4.ERR_ALIAS  # y over x
    assert call(ws=0x100000) == gq4.ERR_ALIAS  # workspace over gate weights
    assert call(logits=0) == gq4.ERR_NULL
    assert call(g=_desc(out=F, in_=H, gs=32, w=0x100000, s=0x200000, E=E)) == gq4.ERR_UNSUPPORTED  # MoE: gs 64
    r = gq4.RoutingDesc()
    assert L.moe_expert_ffn_routing(0x800000, ws_bytes, T, E, K, H, F, ctypes.byref(r)) == gq4.OK
    ptrs = [r.idx, r.wts, r.cnt, r.offs, r.row_tok, r.row_slot, r.slot_row, r.n_active, r.active, r.status]
    assert all(p % 16 == 0 and 0x800000 <= p < 0x800000 + ws_bytes for p in ptrs)
    assert len(set(ptrs)) == len(ptrs)


def test_detect_group_size_host():
    L = gq4.lib()
    gs = ctypes.c_int32(0)
    assert L.gq4_detect_group_size(28672, 512, 917504, ctypes.byref(gs)) == gq4.OK and gs.value == 64
    assert L.gq4_detect_group_size(2048, 6144, 2048 * 48 * 4, ctypes.byref(gs)) == gq4.OK and gs.value == 128
    assert L.gq4_detect_group_size(100, 4096, 123, ctypes.byref(gs)) == gq4.ERR_SHAPE
    assert L.gq4_detect_group_size(100, 16, 400, ctypes.byref(gs)) == gq4.ERR_UNSUPPORTED
    assert L.gq4_detect_group_size(100, 16, 400, None) == gq4.ERR_NULL
    assert gq4.detect_group_size(6144, 2048, 6144 * 32 * 4) == 64


def test_quantize_and_row_ops_argument_checks():
    """Every rejected call returns before anything is launched (fake pointers)."""
    L = gq4.lib()
    d = gq4.TensorDesc()
    q = lambda w=0x100000, O=64, I=128, gs=64, dw=0x200000, dwb=4096, ds=0x300000, dsb=512: \
        L.gq4_quantize(w, O, I, gs, dw, dwb, ds, dsb, None, ctypes.byref(d))
    assert q(w=0) == gq4.ERR_NULL
    assert q(gs=12) == gq4.ERR_UNSUPPORTED
    assert q(I=100) == gq4.ERR_UNSUPPORTED
    assert q(dwb=4095) == gq4.ERR_SHAPE
    assert q(w=0x100004) == gq4.ERR_ALIGN
    assert q(dw=0x100000) == gq4.ERR_ALIAS
    W = _desc()
    dr = lambda idx=0x500000, n=3, alpha=None, acc=0, out=0x600000, odt=0, d=W: \
        L.gq4_dequant_rows(ctypes.byref(d), idx, n, alpha, acc, out, odt, None)
    assert dr(idx=0) == gq4.ERR_NULL
    assert dr(n=0) == gq4.ERR_SHAPE
    assert dr(odt=1, acc=1) == gq4.ERR_UNSUPPORTED
    assert dr(out=0x600008) == gq4.ERR_ALIGN
    assert dr(out=0x10000) == gq4.ERR_ALIAS
    assert dr(d=_desc(gs=12)) == gq4.ERR_UNSUPPORTED
    mr = lambda idx=0x500000, n=3, x=0x700000, xdt=1, T=1, y=0x800000: \
        L.gq4_matvec_rows(ctypes.byref(W), idx, n, x, xdt, T, y, None)
    assert mr(x=0) == gq4.ERR_NULL
    assert mr(T=0) == gq4.ERR_SHAPE
    assert mr(xdt=5) == gq4.ERR_UNSUPPORTED
    assert mr(y=0x700000) == gq4.ERR_ALIAS
    assert mr(idx=0x500002) == gq4.ERR_ALIGN


def test_mla_absorb_argument_checks():
    """Rejected MLA absorb calls return before anything is launched (fake pointers)."""
    L = gq4.lib()
    W = _desc(out=2 * (16 + 48), in_=512)
    for fn in (L.gq4_mla_absorb_q, L.gq4_mla_absorb_v):
        c = lambda nh=2, dn=16, dv=48, x=0x700000, dt=1, T=3, out=0x900000, d=W: \
            fn(ctypes.byref(d), nh, dn, dv, x, dt, T, out, None)
        assert c(x=0) == gq4.ERR_NULL
        assert c(out=0) == gq4.ERR_NULL
        assert c(dv=47) == gq4.ERR_SHAPE           # n_heads * (d_nope + d_v) != out
        assert c(nh=0) == gq4.ERR_SHAPE
        assert c(T=0) == gq4.ERR_SHAPE
        assert c(T=4 * 65536) == gq4.ERR_SHAPE
        assert c(dt=7) == gq4.ERR_UNSUPPORTED
        assert c(d=_desc(out=2 * (16 + 48), in_=4096)) == gq4.ERR_UNSUPPORTED  # R > 2048
        assert c(dn=1040, dv=-976) == gq4.ERR_SHAPE
        assert c(x=0x700004) == gq4.ERR_ALIGN
        assert c(out=0x700000) == gq4.ERR_ALIAS
    big = _desc(out=1025 + 7, in_=64)
    assert L.gq4_mla_absorb_q(ctypes.byref(big), 1, 1025, 7, 0x700000, 0, 1, 0x900000, None) == gq4.ERR_UNSUPPORTED


def test_wait_selftest_argument_checks():
    """The wait self-test refuses bad arguments before launching (fake pointers)."""
    L = gq4.lib()
    assert L.gq4_selftest_wait_timeout(1000, None, None) == gq4.ERR_NULL
    assert L.gq4_selftest_wait_timeout(1000, 0x100004, None) == gq4.ERR_ALIGN
    assert L.gq4_selftest_wait_timeout(0, 0x100000, None) == gq4.ERR_SHAPE
    assert L.gq4_selftest_wait_timeout(2000000, 0x100000, None) == gq4.ERR_SHAPE


def test_sync_status_argument_checks():
    """gq4_sync_status refuses null or misaligned pointers before any CUDA call."""
    L = gq4.lib()
    v = ctypes.c_int32(-1)
    assert L.gq4_sync_status(None, None, ctypes.byref(v)) == gq4.ERR_NULL
    assert L.gq4_sync_status(0x100000, None, None) == gq4.ERR_NULL
    assert L.gq4_sync_status(0x100004, None, ctypes.byref(v)) == gq4.ERR_ALIGN
    assert v.value == -1


def test_checked_library_loads_and_exports_every_symbol():
    """The bounds-checked build exports the same ABI and says it is checked (host calls
    only; no GPU needed)."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    lib = os.path.join(root, "weight_only_int4_gq4_b200", "libgq4_checked.so")
    assert os.path.exists(lib), "build it with `python -m weight_only_int4_gq4_b200.build --checked`"
    code = ("from weight_only_int4_gq4_b200 import gq4\n"
            "assert gq4.build_checked() == 1\n"
            "assert all(hasattr(gq4.lib(), n) for n in gq4.EXPORTED)\n"
            "print('ok')\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env=dict(os.environ, GQ4_LIBRARY=lib),
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr
