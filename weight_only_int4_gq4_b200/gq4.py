"""Thin Python binding over libgq4.so (the C ABI in include/gq4.h).

Argument marshalling only: every step of the computation runs in the CUDA kernels of
the library.  PyTorch provides device memory and the current CUDA stream.  Importing
this module loads the library and raises if it is missing or of another ABI version;
there is no fallback.  GQ4_LIBRARY, when set, names another build of the same library to
load instead (the bounds-checked build, libgq4_checked.so).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("GQ4_LIBRARY") or os.path.join(_HERE, "libgq4.so")
CHECKED_LIB_PATH = os.path.join(_HERE, "libgq4_checked.so")
ABI_VERSION = 7
MOE_STAGE_EVENTS = 6
MOE_LARGE_MIN_ROWS = 33  # GQ4_MOE_LARGE_MIN_ROWS
NOALLOC_SCRATCH_BYTES = 16 << 20  # GQ4_NOALLOC_SCRATCH_BYTES

OK, ERR_NULL, ERR_ALIGN, ERR_SHAPE, ERR_UNSUPPORTED, ERR_ALIAS, ERR_WORKSPACE, ERR_CUDA, \
    ERR_TIMEOUT, ERR_NONFINITE_LOGIT = range(10)
ERR_BOUNDS = 16
F32, BF16 = 0, 1

if not os.path.exists(LIB_PATH):
    raise RuntimeError(
        f"{os.path.basename(LIB_PATH)} not found at {LIB_PATH}: build it with "
        "`python -m weight_only_int4_gq4_b200.build` (nvcc, sm_100a)")
_lib = ctypes.CDLL(LIB_PATH)


class TensorDesc(ctypes.Structure):
    _fields_ = [("out", ctypes.c_int64), ("in_", ctypes.c_int64), ("gs", ctypes.c_int32),
                ("ng", ctypes.c_int32), ("n_experts", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("w", ctypes.c_void_p), ("s", ctypes.c_void_p),
                ("expert_stride_w", ctypes.c_int64), ("expert_stride_s", ctypes.c_int64)]


class RoutingDesc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("idx", "wts", "cnt", "offs", "row_tok", "row_slot", "slot_row", "n_active",
                 "active", "status", "h")]


_P, _I64, _I32, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
_TP = ctypes.POINTER(TensorDesc)
_SIGS = {
    "gq4_abi_version": ([], ctypes.c_uint32),
    "gq4_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "gq4_pack": ([_P, _I64, _I64, _I32, _I32, _P], ctypes.c_int),
    "gq4_device_bytes": ([_I64, _I64, _I32, _I32, ctypes.POINTER(_SZ), ctypes.POINTER(_SZ)], ctypes.c_int),
    "gq4_upload": ([_P, _P, _I64, _I64, _I32, _I32, _I32, _P, _SZ, _P, _SZ, _P, _TP], ctypes.c_int),
    "gq4_tensor_init": ([_P, _P, _I64, _I64, _I32, _I32, _TP], ctypes.c_int),
    "gq4_matvec": ([_TP, _P, ctypes.c_int, _I64, _P, _P], ctypes.c_int),
    "gq4_gate_up_silu": ([_TP, _TP, _P, ctypes.c_int, _I64, _P, _P], ctypes.c_int),
    "gq4_route": ([_P, _I64, _I32, _I32, _P, _P, _P, _P], ctypes.c_int),
    "gq4_rowmap_scratch_bytes": ([_I64, _I32, _I32], _SZ),
    "gq4_rowmap": ([_P, _I64, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "moe_expert_ffn_workspace_bytes": ([_I64, _I32, _I32, _I64, _I64], _SZ),
    "moe_expert_ffn": ([_TP, _TP, _TP, _P, _P, ctypes.c_int, _I64, _I32, _I32, _P, _P, _SZ, _P, _P],
                       ctypes.c_int),
    "moe_expert_ffn_routing": ([_P, _SZ, _I64, _I32, _I32, _I64, _I64, ctypes.POINTER(RoutingDesc)],
                               ctypes.c_int),
    "moe_expert_ffn_status": ([_P, _SZ, _I64, _I32, _I32, _I64, _I64, _P, ctypes.POINTER(_I32)],
                              ctypes.c_int),
    "moe_expert_ffn_noalloc": ([_TP, _TP, _TP, _P, _P, ctypes.c_int, _I64, _I32, _I32, _P, _P, _P],
                               ctypes.c_int),
    "gq4_detect_group_size": ([_I64, _I64, _SZ, ctypes.POINTER(_I32)], ctypes.c_int),
    "gq4_quantize": ([_P, _I64, _I64, _I32, _P, _SZ, _P, _SZ, _P, _TP], ctypes.c_int),
    "gq4_dequant_rows": ([_TP, _P, _I64, _P, _I32, _P, ctypes.c_int, _P], ctypes.c_int),
    "gq4_matvec_rows": ([_TP, _P, _I64, _P, ctypes.c_int, _I64, _P, _P], ctypes.c_int),
    "gq4_mla_absorb_q": ([_TP, _I32, _I32, _I32, _P, ctypes.c_int, _I64, _P, _P], ctypes.c_int),
    "gq4_mla_absorb_v": ([_TP, _I32, _I32, _I32, _P, ctypes.c_int, _I64, _P, _P], ctypes.c_int),
    "gq4_selftest_wait_timeout": ([ctypes.c_uint32, _P, _P], ctypes.c_int),
    "gq4_sync_status": ([_P, _P, ctypes.POINTER(_I32)], ctypes.c_int),
    "gq4_build_checked": ([], ctypes.c_int32),
    "gq4_bounds_status": ([_I32, _P, ctypes.POINTER(_I32)], ctypes.c_int),
    "gq4_selftest_bounds": ([_I64, _I64, _P], ctypes.c_int),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res

if _lib.gq4_abi_version() != ABI_VERSION:
    raise RuntimeError(f"libgq4 ABI {_lib.gq4_abi_version()} != binding ABI {ABI_VERSION}; rebuild")

EXPORTED = tuple(_SIGS)


class GQ4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.gq4_status_string(status).decode()} (status {status})")


def _check(st: int, where: str):
    if st != OK:
        raise GQ4Error(st, where)


def lib() -> ctypes.CDLL:
    return _lib


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _xdt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"activations must be float32 or bfloat16, got {t.dtype}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("expected contiguous CUDA tensors")


# ------------------------------------------------------------------ host packing
def pack(q: np.ndarray, gs: int = 64, offset_binary: bool = False) -> np.ndarray:
    """int8 q [O][I] (-8..7, or 0..15 offset-binary) -> packed uint8 [O][ceil(I/2)]."""
    q = np.ascontiguousarray(q, np.int8)
    O, I = q.shape
    out = np.empty((O, (I + 1) // 2), np.uint8)
    _check(_lib.gq4_pack(q.ctypes.data, O, I, gs, int(offset_binary), out.ctypes.data), "gq4_pack")
    return out


def device_bytes(out: int, in_: int, gs: int = 64, n_experts: int = 1):
    w, s = _SZ(), _SZ()
    _check(_lib.gq4_device_bytes(out, in_, gs, n_experts, ctypes.byref(w), ctypes.byref(s)),
           "gq4_device_bytes")
    return w.value, s.value


@dataclass
class Tensor:
    """A grouped-int4 matrix (or a stack of experts) resident on the GPU."""
    desc: TensorDesc
    w: torch.Tensor  # uint8 device storage
    s: torch.Tensor  # float32 device storage

    @property
    def out(self):
        return self.desc.out

    @property
    def in_(self):
        return self.desc.in_

    def ref(self):
        return ctypes.byref(self.desc)


def upload(packed: np.ndarray, scales: np.ndarray, gs: int = 64, offset_binary: bool = False,
           device="cuda", stream=None) -> Tensor:
    """packed uint8 [(E,) O, ceil(I/2)] and scales f32 [(E,) O, ng] -> Tensor on the GPU.

    The host arrays are copied with gq4_upload on the current stream; the call
    synchronises that stream before returning so numpy buffers may be released."""
    packed = np.ascontiguousarray(packed, np.uint8)
    scales = np.ascontiguousarray(scales, np.float32)
    if packed.ndim == 2:
        packed, scales = packed[None], scales[None]
    E, O, rb = packed.shape
    ng = scales.shape[2]
    I = ng * gs if (ng * gs + 1) // 2 == rb else 2 * rb
    wb, sb = device_bytes(O, I, gs, E)
    if packed.nbytes != wb or scales.nbytes != sb:
        raise ValueError("packed/scales sizes do not match the grouped-int4 layout")
    d_w = torch.empty(wb, dtype=torch.uint8, device=device)
    d_s = torch.empty(sb // 4, dtype=torch.float32, device=device)
    desc = TensorDesc()
    st = _stream(stream)
    _check(_lib.gq4_upload(packed.ctypes.data, scales.ctypes.data, O, I, gs, E, int(offset_binary),
                           d_w.data_ptr(), wb, d_s.data_ptr(), sb, st, ctypes.byref(desc)),
           "gq4_upload")
    torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()
    return Tensor(desc, d_w, d_s)


def from_device(d_w: torch.Tensor, d_s: torch.Tensor, out: int, in_: int, gs: int = 64,
                n_experts: int = 1) -> Tensor:
    desc = TensorDesc()
    _check(_lib.gq4_tensor_init(d_w.data_ptr(), d_s.data_ptr(), out, in_, gs, n_experts,
                                ctypes.byref(desc)), "gq4_tensor_init")
    return Tensor(desc, d_w, d_s)


# ------------------------------------------------------------------ compute
def matvec(W: Tensor, x: torch.Tensor, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y [T][O] f32 = x [T][I] (f32 or bf16) times W^T."""
    if x.dim() == 1:
        x = x[None]
    if y is None:
        y = torch.empty(x.shape[0], W.out, dtype=torch.float32, device=x.device)
    _need_cuda(x, y)
    _check(_lib.gq4_matvec(W.ref(), x.data_ptr(), _xdt(x), x.shape[0], y.data_ptr(), _stream(stream)),
           "gq4_matvec")
    return y


def gate_up_silu(Wg: Tensor, Wu: Tensor, x: torch.Tensor, h: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    """h [T][F] (x's dtype) = silu(Wg x) * (Wu x), x read once."""
    if x.dim() == 1:
        x = x[None]
    if h is None:
        h = torch.empty(x.shape[0], Wg.out, dtype=x.dtype, device=x.device)
    _need_cuda(x, h)
    _check(_lib.gq4_gate_up_silu(Wg.ref(), Wu.ref(), x.data_ptr(), _xdt(x), x.shape[0], h.data_ptr(),
                                 _stream(stream)), "gq4_gate_up_silu")
    return h


def route(logits: torch.Tensor, K: int, stream=None):
    """-> (idx int32 [T][K], wts f32 [T][K], status int32 [1]) on the device."""
    T, E = logits.shape
    dev = logits.device
    idx = torch.empty(T, K, dtype=torch.int32, device=dev)
    wts = torch.empty(T, K, dtype=torch.float32, device=dev)
    status = torch.zeros(4, dtype=torch.int32, device=dev)
    _need_cuda(logits)
    _check(_lib.gq4_route(logits.data_ptr(), T, E, K, idx.data_ptr(), wts.data_ptr(), status.data_ptr(),
                          _stream(stream)), "gq4_route")
    return idx, wts, status[:1]


def rowmap(idx: torch.Tensor, E: int, stream=None):
    """-> dict of device int32 tensors: cnt, offs, row_tok, row_slot, slot_row, n_active,
    active, status."""
    T, K = idx.shape
    dev = idx.device
    n = T * K
    out = {k: torch.empty(sz, dtype=torch.int32, device=dev) for k, sz in
           (("cnt", E), ("offs", E + 1), ("row_tok", n), ("row_slot", n), ("slot_row", n),
            ("n_active", 4), ("active", E))}
    sb = _lib.gq4_rowmap_scratch_bytes(T, K, E)
    scratch = torch.empty(sb, dtype=torch.uint8, device=dev)
    _need_cuda(idx)
    _check(_lib.gq4_rowmap(idx.data_ptr(), T, K, E, out["cnt"].data_ptr(), out["offs"].data_ptr(),
                           out["row_tok"].data_ptr(), out["row_slot"].data_ptr(),
                           out["slot_row"].data_ptr(), out["n_active"].data_ptr(),
                           out["active"].data_ptr(), scratch.data_ptr(), sb, _stream(stream)),
           "gq4_rowmap")
    out["n_active"] = out["n_active"][:1]
    out["status"] = scratch[:4].view(torch.int32)
    return out


def moe_workspace_bytes(T: int, E: int, K: int, H: int, F: int) -> int:
    return _lib.moe_expert_ffn_workspace_bytes(T, E, K, H, F)


class MoEWorkspace:
    """Device workspace of moe_expert_ffn for one (T, E, K, H, F)."""

    def __init__(self, T, E, K, H, F, device="cuda"):
        self.shape = (T, E, K, H, F)
        self.nbytes = moe_workspace_bytes(T, E, K, H, F)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)

    def routing(self) -> dict:
        """Views of the routing tables (device int32/f32 tensors) and of h (bf16 bit
        patterns as int16, [T*K][F], row-map order) after a call."""
        T, E, K, H, F = self.shape
        r = RoutingDesc()
        _check(_lib.moe_expert_ffn_routing(self.buf.data_ptr(), self.nbytes, T, E, K, H, F,
                                           ctypes.byref(r)), "moe_expert_ffn_routing")
        base = self.buf.data_ptr()
        n = T * K

        def view(ptr, count, dtype):
            off = ptr - base
            esz = 4
            return self.buf[off:off + count * esz].view(dtype)

        return dict(idx=view(r.idx, n, torch.int32).view(T, K), wts=view(r.wts, n, torch.float32).view(T, K),
                    cnt=view(r.cnt, E, torch.int32), offs=view(r.offs, E + 1, torch.int32),
                    row_tok=view(r.row_tok, n, torch.int32), row_slot=view(r.row_slot, n, torch.int32),
                    slot_row=view(r.slot_row, n, torch.int32), n_active=view(r.n_active, 1, torch.int32),
                    active=view(r.active, E, torch.int32), status=view(r.status, 1, torch.int32),
                    h=self.buf[r.h - base:r.h - base + n * F * 2].view(torch.int16).view(n, F))

    def status(self, stream=None) -> int:
        T, E, K, H, F = self.shape
        v = _I32()
        _check(_lib.moe_expert_ffn_status(self.buf.data_ptr(), self.nbytes, T, E, K, H, F,
                                          _stream(stream), ctypes.byref(v)), "moe_expert_ffn_status")
        return v.value


def moe_expert_ffn(Wg: Tensor, Wu: Tensor, Wd: Tensor, logits: torch.Tensor, x: torch.Tensor, K: int,
                   y: torch.Tensor | None = None, ws: MoEWorkspace | None = None, stream=None,
                   stage_events=None):
    """y [T][H] f32 for one routed-expert FFN layer (x bf16 [T][H], logits f32 [T][E]).

    stage_events: optional 6 torch.cuda.Event(enable_timing=True) recorded at the start,
    after routing, after gate+up of the experts with few rows, after gate+up of those
    with many rows, after down of the few-row experts and after down of the others."""
    T, H = x.shape
    E = logits.shape[1]
    F = Wg.out
    if ws is None:
        ws = MoEWorkspace(T, E, K, H, F, device=x.device)
    if y is None:
        y = torch.empty(T, H, dtype=torch.float32, device=x.device)
    _need_cuda(x, logits, y)
    ev = None
    if stage_events is not None:
        if len(stage_events) != MOE_STAGE_EVENTS:
            raise ValueError(f"stage_events: {MOE_STAGE_EVENTS} events expected")
        ev = (ctypes.c_void_p * MOE_STAGE_EVENTS)(*[e.cuda_event for e in stage_events])
    _check(_lib.moe_expert_ffn(Wg.ref(), Wu.ref(), Wd.ref(), logits.data_ptr(), x.data_ptr(), _xdt(x),
                               T, E, K, y.data_ptr(), ws.buf.data_ptr(), ws.nbytes, ev, _stream(stream)),
           "moe_expert_ffn")
    return y, ws


def moe_expert_ffn_noalloc(Wg: Tensor, Wu: Tensor, Wd: Tensor, logits: torch.Tensor, x: torch.Tensor,
                           K: int, y: torch.Tensor, status_out: torch.Tensor | None = None, stream=None):
    """moe_expert_ffn without a workspace, for callers that cannot allocate device memory.

    The library's own device array (NOALLOC_SCRATCH_BYTES per GPU) replaces the
    workspace; y (and status_out, a device int32 tensor of at least one element, if given)
    are the caller's.  Calls that overlap on the GPU share that array and race: serialise
    them."""
    T, H = x.shape
    E = logits.shape[1]
    _need_cuda(x, logits, y, status_out)
    _check(_lib.moe_expert_ffn_noalloc(Wg.ref(), Wu.ref(), Wd.ref(), logits.data_ptr(), x.data_ptr(),
                                       _xdt(x), T, E, K, y.data_ptr(), _ptr(status_out), _stream(stream)),
           "moe_expert_ffn_noalloc")
    return y


# ------------------------------------------------------------------ general group sizes, rows
def detect_group_size(out: int, in_: int, scale_bytes: int) -> int:
    """Group size of a matrix from its scale array's byte count (raises if none or ambiguous)."""
    gs = _I32()
    _check(_lib.gq4_detect_group_size(out, in_, scale_bytes, ctypes.byref(gs)), "gq4_detect_group_size")
    return gs.value


def quantize(w: torch.Tensor, gs: int = 64, stream=None) -> Tensor:
    """f32 device weights [O][I] -> grouped-int4 Tensor (absmax scales, round half to even)."""
    if w.dtype != torch.float32 or w.dim() != 2:
        raise TypeError("quantize: expected a 2-D float32 tensor")
    _need_cuda(w)
    O, I = w.shape
    wb, sb = device_bytes(O, I, gs, 1)
    d_w = torch.empty(wb, dtype=torch.uint8, device=w.device)
    d_s = torch.empty(sb // 4, dtype=torch.float32, device=w.device)
    desc = TensorDesc()
    _check(_lib.gq4_quantize(w.data_ptr(), O, I, gs, d_w.data_ptr(), wb, d_s.data_ptr(), sb, _stream(stream),
                             ctypes.byref(desc)), "gq4_quantize")
    return Tensor(desc, d_w, d_s)


def dequant_rows(W: Tensor, idx: torch.Tensor, alpha: torch.Tensor | None = None, out: torch.Tensor | None = None,
                 accumulate: bool = False, dtype=torch.float32, stream=None) -> torch.Tensor:
    """out [n][I] = (accumulate ? out : 0) + alpha[j] * w[idx[j]] (rows dequantised)."""
    n = idx.shape[0]
    if out is None:
        out = torch.empty(n, W.in_, dtype=dtype, device=idx.device)
    _need_cuda(idx, out, alpha)
    odt = _xdt(out)
    _check(_lib.gq4_dequant_rows(W.ref(), idx.data_ptr(), n, _ptr(alpha), int(accumulate), out.data_ptr(), odt,
                                 _stream(stream)), "gq4_dequant_rows")
    return out


def matvec_rows(W: Tensor, idx: torch.Tensor, x: torch.Tensor, y: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
    """y [T][n] f32 = x [T][I] times the selected rows of W."""
    if x.dim() == 1:
        x = x[None]
    n = idx.shape[0]
    if y is None:
        y = torch.empty(x.shape[0], n, dtype=torch.float32, device=x.device)
    _need_cuda(idx, x, y)
    _check(_lib.gq4_matvec_rows(W.ref(), idx.data_ptr(), n, x.data_ptr(), _xdt(x), x.shape[0], y.data_ptr(),
                                _stream(stream)), "gq4_matvec_rows")
    return y


def mla_absorb_q(W: Tensor, n_heads: int, d_nope: int, d_v: int, q_nope: torch.Tensor,
                 q_lat: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """q_lat [T][n_heads][R] f32 = q_nope [T][n_heads][d_nope] times each head's key rows
    of the kv_b tensor W (rows in per-head blocks of d_nope key + d_v value rows)."""
    T = q_nope.shape[0]
    if q_lat is None:
        q_lat = torch.empty(T, n_heads, W.in_, dtype=torch.float32, device=q_nope.device)
    _need_cuda(q_nope, q_lat)
    _check(_lib.gq4_mla_absorb_q(W.ref(), n_heads, d_nope, d_v, q_nope.data_ptr(), _xdt(q_nope), T,
                                 q_lat.data_ptr(), _stream(stream)), "gq4_mla_absorb_q")
    return q_lat


def mla_absorb_v(W: Tensor, n_heads: int, d_nope: int, d_v: int, lat: torch.Tensor,
                 o: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """o [T][n_heads][d_v] f32 = lat [T][n_heads][R] times each head's value rows of the
    kv_b tensor W."""
    T = lat.shape[0]
    if o is None:
        o = torch.empty(T, n_heads, d_v, dtype=torch.float32, device=lat.device)
    _need_cuda(lat, o)
    _check(_lib.gq4_mla_absorb_v(W.ref(), n_heads, d_nope, d_v, lat.data_ptr(), _xdt(lat), T,
                                 o.data_ptr(), _stream(stream)), "gq4_mla_absorb_v")
    return o


def selftest_wait_timeout(limit_us: int = 1000, stream=None) -> int:
    """Runs the kernels' bounded wait on a barrier nothing completes; returns the status
    word it leaves (GQ4_ERR_TIMEOUT when the wait gave up as designed)."""
    st = torch.zeros(4, dtype=torch.int32, device="cuda")
    _check(_lib.gq4_selftest_wait_timeout(limit_us, st.data_ptr(), _stream(stream)), "gq4_selftest_wait_timeout")
    return sync_status(st, stream)


def sync_status(status: torch.Tensor, stream=None) -> int:
    """Waits for the stream and returns the device status word status[0]."""
    _need_cuda(status)
    v = _I32()
    _check(_lib.gq4_sync_status(status.data_ptr(), _stream(stream), ctypes.byref(v)), "gq4_sync_status")
    return v.value


# ------------------------------------------------------------------ checked build
def build_checked() -> bool:
    """True when the loaded library is the bounds-checked build."""
    return bool(_lib.gq4_build_checked())


def bounds_status(clear: bool = True, stream=None) -> int:
    """Waits for the stream and returns the bounds status word (0 or ERR_BOUNDS)."""
    v = _I32()
    _check(_lib.gq4_bounds_status(int(clear), _stream(stream), ctypes.byref(v)), "gq4_bounds_status")
    return v.value


def selftest_bounds(index: int, extent: int, stream=None) -> None:
    """Tests index against extent on the device without any memory access."""
    _check(_lib.gq4_selftest_bounds(index, extent, _stream(stream)), "gq4_selftest_bounds")
