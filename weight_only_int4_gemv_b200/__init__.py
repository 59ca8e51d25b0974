"""Python binding of libawq_b200: a W4A16 (group-wise INT4 weight, fp16
activation) linear layer for NVIDIA B200.

Every function marshals torch tensors into the C ABI declared in
``include/awq.h`` and enqueues the library's CUDA kernels on the current
torch stream. Nothing here computes: there is no CPU fallback, and using the
binding without the built library or without a CUDA device raises.

Layouts (row-major, K contiguous): W fp16 [N, K]; x fp16 [M, K]; y fp16
[M, N]; qweight int32 [N, K/8] (eight 4-bit codes per word, nibble slot i of
word w holds k = 8w + (0, 2, 4, 6, 1, 3, 5, 7)[i]); scales fp16 [K/128, N];
zeros fp16 [K/128, N] holding integers 0..15 (None for the symmetric
variant, whose zero point is 8); scales and zeros are group-major.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "LIB_PATH", "AwqError", "lib", "GROUP_SIZE",
    "awq_pseudo_quantize_pack", "awq_dequant", "awq_workspace_bytes",
    "awq_gemv", "awq_gemm", "awq_device_error", "awq_linear", "GEMV_MAX_M", "awq_gemv_noalloc",
    "awq_pack_zeros", "awq_unpack_zeros", "validate_product", "GemvChain", "awq_gemv_chain",
    "CHAIN_MAX_LAYERS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libawq_b200.so")
GROUP_SIZE = 128
GEMV_MAX_M = 16

AWQ_OK = 0
STATUS_NAMES = {0: "AWQ_OK", 1: "AWQ_ERR_NULL", 2: "AWQ_ERR_SHAPE", 3: "AWQ_ERR_ALIGN",
                4: "AWQ_ERR_UNSUPPORTED", 5: "AWQ_ERR_CUDA", 6: "AWQ_ERR_WORKSPACE"}


class AwqError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)} ({text})")
        self.status = status


ABI_VERSION = 8   # awq_abi_version() of a library this binding matches


class QConfig(ctypes.Structure):
    _fields_ = [("group_size", ctypes.c_int32), ("zero_point", ctypes.c_int32), ("flags", ctypes.c_uint32)]


# awq_qconfig_t.flags bit: qweight / scales / zeros are not written by work
# still running on the stream, so the GEMV may read them before the previous
# kernel finishes (it still waits for that kernel before reading x).
FLAG_WEIGHTS_STATIC = 1
FLAG_SILU_MUL = 2   # rows are 16-row tiles alternating gate, up; y = silu(gate) * up, N/2 columns
FLAG_PACKED_ZEROS = 4   # zeros is int32 qzeros [K/128, N/8], eight 4-bit zero points per word


class GemvLayer(ctypes.Structure):
    """awq_gemv_layer_t: one layer of an awq_gemv_chain call."""
    _fields_ = [("x", ctypes.c_void_p), ("qweight", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("zeros", ctypes.c_void_p), ("y", ctypes.c_void_p), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64), ("cfg", QConfig), ("x_from", ctypes.c_int32)]


CHAIN_MAX_LAYERS = 32

_lib = None
_lock = threading.Lock()

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SIGS = {
    "awq_abi_version": (ctypes.c_int, []),
    "awq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "awq_pseudo_quantize_pack": (ctypes.c_int, [_P, _I64, _I64, QConfig, _P, _P, _P, _P]),
    "awq_dequant": (ctypes.c_int, [_P, _P, _P, _I64, _I64, QConfig, _P, _P]),
    "awq_workspace_bytes": (ctypes.c_int, [_I64, _I64, _I64, QConfig, ctypes.POINTER(ctypes.c_size_t)]),
    "awq_gemv": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, QConfig, _P, _P, ctypes.c_size_t, _P]),
    "awq_gemm": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, QConfig, _P, _P, ctypes.c_size_t, _P]),
    "awq_device_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), _P]),
    "awq_gemv_noalloc": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, QConfig, _P, _P]),
    "awq_pack_zeros": (ctypes.c_int, [_P, _I64, _I64, _P, _P]),
    "awq_unpack_zeros": (ctypes.c_int, [_P, _I64, _I64, _P, _P]),
    "awq_interleave_gate_up": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, QConfig, _P, _P, _P, _P]),
    "awq_concat_rows": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(_P),
                                       ctypes.POINTER(_I64), _I64, QConfig, _P, _P, _P, _P]),
    "awq_search_scale_workspace_bytes": (ctypes.c_int, [_I64, _I64, _I64, QConfig, ctypes.POINTER(ctypes.c_size_t)]),
    "awq_search_scale": (ctypes.c_int, [_P, _I64, _I64, _P, _I64, QConfig, ctypes.c_int, ctypes.c_int, _P, _P, _P,
                                        ctypes.c_size_t, _P]),
    "awq_apply_scale": (ctypes.c_int, [_P, _P, _I64, _I64, _P, _P]),
    "awq_search_clip_workspace_bytes": (ctypes.c_int, [_I64, ctypes.POINTER(ctypes.c_size_t)]),
    "awq_search_clip": (ctypes.c_int, [_P, _I64, _I64, _P, _I64, QConfig, ctypes.c_int, ctypes.c_float, _P, _P,
                                       ctypes.c_size_t, _P]),
    "awq_apply_clip": (ctypes.c_int, [_P, _P, _I64, _I64, _P, _P]),
    "awq_gemv_chain_workspace_bytes": (ctypes.c_int, [ctypes.POINTER(GemvLayer), ctypes.c_int, _I64,
                                                      ctypes.POINTER(ctypes.c_size_t)]),
    "awq_gemv_chain": (ctypes.c_int, [ctypes.POINTER(GemvLayer), ctypes.c_int, _I64, _P, ctypes.c_size_t, _P]),
    "awq_debug_set_wait_limit_ns": (ctypes.c_int, [ctypes.c_uint64, _P]),
}


def lib():
    """The loaded shared library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        f"{LIB_PATH} is missing: build it with "
                        "`python -m weight_only_int4_gemv_b200.build` (there is no fallback)")
                h = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in _SIGS.items():
                    f = getattr(h, name)
                    f.restype = res
                    f.argtypes = args
                if h.awq_abi_version() != ABI_VERSION:
                    raise RuntimeError(f"{LIB_PATH} has ABI version {h.awq_abi_version()}, this binding "
                                       f"needs {ABI_VERSION}: rebuild it")
                _lib = h
    return _lib


def _check(fn: str, st: int):
    if st != AWQ_OK:
        raise AwqError(fn, st, lib().awq_status_string(st).decode())


_CFGS = {}


def _cfg(zero_point: bool, group_size: int, flags: int = 0) -> QConfig:
    key = (bool(zero_point), group_size, flags)
    c = _CFGS.get(key)
    if c is None:
        c = _CFGS[key] = QConfig(group_size, 1 if zero_point else 0, flags)
    return c


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _form(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int):
    """Type, dtype, rank and contiguity of one operand (no device check)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-d tensor")


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int):
    if isinstance(t, torch.Tensor) and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
    _form(t, name, dtype, ndim)


def _same_device(ref: torch.Tensor, **tensors):
    """Every given tensor (None skipped) must sit on ref's device."""
    for name, t in tensors.items():
        if t is not None and t.device != ref.device:
            raise ValueError(f"{name} is on {t.device}, expected {ref.device}: operands must share a device")


def _out_shape(out: torch.Tensor, shape):
    if tuple(out.shape) != tuple(shape):
        raise ValueError(f"out must be {list(shape)}, got {list(out.shape)}")


def _zeros_flag(zeros, N: int, K: int, group_size: int) -> int:
    """Check the zero points' form: fp16 [K/g, N], or int32 qzeros [K/g, N/8]
    (AWQ_FLAG_PACKED_ZEROS, returned as the flag to pass)."""
    if zeros is None:
        return 0
    if isinstance(zeros, torch.Tensor) and zeros.dtype == torch.int32:
        _form(zeros, "zeros", torch.int32, 2)
        if group_size == GROUP_SIZE and (N % 8 or zeros.shape != (K // group_size, N // 8)):
            raise ValueError("packed zeros must be int32 [K/group_size, N/8]")
        return FLAG_PACKED_ZEROS
    _form(zeros, "zeros", torch.float16, 2)
    if group_size == GROUP_SIZE and zeros.shape != (K // group_size, N):
        raise ValueError("scales / zeros must be [K/group_size, N]")
    return 0


def awq_pack_zeros(zeros: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """fp16 zero points [G, N] -> int32 qzeros [G, N/8] (eight 4-bit values per
    word, channel 8w+i in bits 4i..4i+3), the AWQ_FLAG_PACKED_ZEROS form that
    awq_gemv and awq_dequant accept in place of the fp16 array."""
    _need(zeros, "zeros", torch.float16, 2)
    G, N = zeros.shape
    if out is None:
        out = torch.empty((G, N // 8), dtype=torch.int32, device=zeros.device)
    _need(out, "out", torch.int32, 2)
    if out.shape != (G, N // 8):
        raise ValueError("out must be int32 [G, N/8]")
    _same_device(zeros, out=out)
    with torch.cuda.device(zeros.device):
        _check("awq_pack_zeros", lib().awq_pack_zeros(_ptr(zeros), G, N, _ptr(out), _stream(zeros.device)))
    return out


def awq_unpack_zeros(qzeros: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """int32 qzeros [G, N/8] -> fp16 zero points [G, N] (the integers 0..15)."""
    _need(qzeros, "qzeros", torch.int32, 2)
    G, N = qzeros.shape[0], qzeros.shape[1] * 8
    if out is None:
        out = torch.empty((G, N), dtype=torch.float16, device=qzeros.device)
    _need(out, "out", torch.float16, 2)
    if out.shape != (G, N):
        raise ValueError("out must be fp16 [G, N]")
    _same_device(qzeros, out=out)
    with torch.cuda.device(qzeros.device):
        _check("awq_unpack_zeros", lib().awq_unpack_zeros(_ptr(qzeros), G, N, _ptr(out), _stream(qzeros.device)))
    return out


def awq_pseudo_quantize_pack(W: torch.Tensor, zero_point: bool = True, group_size: int = GROUP_SIZE):
    """Quantize fp16 W[N, K] and pack it: returns (qweight, scales, zeros or None)."""
    _need(W, "W", torch.float16, 2)
    N, K = W.shape
    G = K // group_size if group_size > 0 else 0
    qweight = torch.empty((N, K // 8), dtype=torch.int32, device=W.device)
    scales = torch.empty((G, N), dtype=torch.float16, device=W.device)          # group-major
    zeros = torch.empty((G, N), dtype=torch.float16, device=W.device) if zero_point else None
    with torch.cuda.device(W.device):
        _check("awq_pseudo_quantize_pack", lib().awq_pseudo_quantize_pack(
            _ptr(W), N, K, _cfg(zero_point, group_size), _ptr(qweight), _ptr(scales), _ptr(zeros),
            _stream(W.device)))
    return qweight, scales, zeros


def awq_dequant(qweight: torch.Tensor, scales: torch.Tensor, zeros, group_size: int = GROUP_SIZE,
                out: torch.Tensor | None = None) -> torch.Tensor:
    """Decode packed weights to fp16 W'[N, K] (bit-exact)."""
    _need(qweight, "qweight", torch.int32, 2)
    _need(scales, "scales", torch.float16, 2)
    N, K = qweight.shape[0], qweight.shape[1] * 8
    zflag = _zeros_flag(zeros, N, K, group_size)
    if group_size == GROUP_SIZE and scales.shape != (K // group_size, N):
        raise ValueError("scales / zeros must be [K/group_size, N]")
    if out is None:
        out = torch.empty((N, K), dtype=torch.float16, device=qweight.device)
    _need(out, "out", torch.float16, 2)
    _out_shape(out, (N, K))
    _same_device(qweight, scales=scales, zeros=zeros, out=out)
    with torch.cuda.device(qweight.device):
        _check("awq_dequant", lib().awq_dequant(
            _ptr(qweight), _ptr(scales), _ptr(zeros), N, K, _cfg(zeros is not None, group_size, zflag),
            _ptr(out), _stream(qweight.device)))
    return out


def awq_workspace_bytes(M: int, N: int, K: int, zero_point: bool = True, group_size: int = GROUP_SIZE,
                        device=None, silu_mul: bool = False, packed_zeros: bool = False) -> int:
    """Workspace bytes awq_gemv / awq_gemm need on `device` for this shape
    (silu_mul: the fused gate/up layout, N = both projections' rows;
    packed_zeros: int32 qzeros; the GEMM unpacks them into its workspace)."""
    n = ctypes.c_size_t(0)
    flags = (FLAG_SILU_MUL if silu_mul else 0) | (FLAG_PACKED_ZEROS if packed_zeros else 0)
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        _check("awq_workspace_bytes", lib().awq_workspace_bytes(
            M, N, K, _cfg(zero_point, group_size, flags), ctypes.byref(n)))
    return int(n.value)


def alloc_workspace(M: int, N: int, K: int, zero_point: bool = True, device=None,
                    silu_mul: bool = False, packed_zeros: bool = False) -> torch.Tensor | None:
    """Zero-filled workspace for (M, N, K), or None when none is needed."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    nbytes = awq_workspace_bytes(M, N, K, zero_point, device=dev, silu_mul=silu_mul, packed_zeros=packed_zeros)
    return torch.zeros(nbytes, dtype=torch.uint8, device=dev) if nbytes else None


def validate_product(x, qweight, scales, zeros, out=None, workspace=None, group_size: int = GROUP_SIZE,
                     flags: int = 0):
    """The host-side checks every product entry point runs before it calls the
    library: dtypes, ranks, contiguity, the shapes of qweight [N, K/8],
    scales [K/g, N], zeros (fp16 [K/g, N] or int32 [K/g, N/8]) and out
    ([M, N], or [M, N/2] with FLAG_SILU_MUL), and that every operand sits on
    x's device. Touches no device. Returns (M, N, K, flags) with the packed
    zero-point flag added when zeros is int32."""
    _form(x, "x", torch.float16, 2)
    _form(qweight, "qweight", torch.int32, 2)
    _form(scales, "scales", torch.float16, 2)
    M, K = x.shape
    N = qweight.shape[0]
    if qweight.shape[1] * 8 != K:
        raise ValueError("qweight must be [N, K/8] for x [M, K]")
    flags |= _zeros_flag(zeros, N, K, group_size)
    if group_size == GROUP_SIZE and scales.shape != (K // group_size, N):
        raise ValueError("scales / zeros must be [K/group_size, N]")
    if out is not None:
        _form(out, "out", torch.float16, 2)
        want = (M, N // 2 if flags & FLAG_SILU_MUL else N)
        if tuple(out.shape) != want:
            raise ValueError(f"out must be [{want[0]}, {want[1]}], got {list(out.shape)}")
    if workspace is not None:
        if not isinstance(workspace, torch.Tensor) or not workspace.is_contiguous():
            raise ValueError("workspace must be a contiguous tensor")
    for name, t in (("qweight", qweight), ("scales", scales), ("zeros", zeros), ("out", out),
                    ("workspace", workspace)):
        if t is not None and t.device != x.device:
            raise ValueError(f"{name} is on {t.device}, x on {x.device}: every operand must be on x's device")
    return M, N, K, flags


def _product(entry: str, x, qweight, scales, zeros, workspace, out, group_size, flags=0):
    _need(x, "x", torch.float16, 2)
    M, N, K, flags = validate_product(x, qweight, scales, zeros, out, workspace, group_size, flags)
    if out is None:
        out = torch.empty((M, N // 2 if flags & FLAG_SILU_MUL else N), dtype=torch.float16, device=x.device)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    fn = getattr(lib(), entry)
    dev = x.device
    args = (_ptr(x), qweight.data_ptr(), scales.data_ptr(), _ptr(zeros), M, N, K,
            _cfg(zeros is not None, group_size, flags), out.data_ptr(), ws_ptr, ws_bytes)
    if dev.index == torch.cuda.current_device():   # no device switch needed (the common case)
        _check(entry, fn(*args, torch.cuda.current_stream().cuda_stream))
    else:
        with torch.cuda.device(dev):
            _check(entry, fn(*args, torch.cuda.current_stream(dev).cuda_stream))
    return out


def _flags(weights_static: bool = False, silu_mul: bool = False) -> int:
    return (FLAG_WEIGHTS_STATIC if weights_static else 0) | (FLAG_SILU_MUL if silu_mul else 0)


def awq_gemv(x, qweight, scales, zeros, workspace=None, out=None, group_size: int = GROUP_SIZE,
             weights_static: bool = False, silu_mul: bool = False):
    """y = x . W'^T for 1 <= M <= 16 (decode). `workspace` from alloc_workspace().
    weights_static: no work still running on the stream writes qweight, scales
    or zeros (a decode loop over loaded weights), so the kernel may start
    streaming them before the previous kernel on the stream has finished.
    silu_mul: the weights are a fused gate/up pair (awq_interleave_gate_up);
    y = silu(x . Wg'^T) * (x . Wu'^T), N/2 columns.
    zeros may be fp16 [K/128, N] or int32 qzeros [K/128, N/8] from
    awq_pack_zeros (N % 32 == 0); y is the same."""
    return _product("awq_gemv", x, qweight, scales, zeros, workspace, out, group_size,
                    _flags(weights_static, silu_mul))


def awq_gemv_noalloc(x, qweight, scales, zeros, out=None, group_size: int = GROUP_SIZE,
                     weights_static: bool = False, silu_mul: bool = False):
    """awq_gemv with the library's fixed scratch array instead of a workspace,
    for callers that cannot allocate device memory when they run the layer.
    Calls on one device share the array and must not overlap on the GPU."""
    _need(x, "x", torch.float16, 2)
    M, N, K, flags = validate_product(x, qweight, scales, zeros, out, None, group_size,
                                      _flags(weights_static, silu_mul))
    if out is None:
        out = torch.empty((M, N // 2 if silu_mul else N), dtype=torch.float16, device=x.device)
    with torch.cuda.device(x.device):
        _check("awq_gemv_noalloc", lib().awq_gemv_noalloc(
            _ptr(x), _ptr(qweight), _ptr(scales), _ptr(zeros), M, N, K,
            _cfg(zeros is not None, group_size, flags), _ptr(out), _stream(x.device)))
    return out


def awq_gemm(x, qweight, scales, zeros, workspace=None, out=None, group_size: int = GROUP_SIZE,
             silu_mul: bool = False):
    """y = x . W'^T for any M (prefill), on the tcgen05 tensor cores.
    silu_mul: as for awq_gemv. zeros may be fp16 [K/128, N] or int32 qzeros
    [K/128, N/8] (N % 32 == 0; the workspace then holds their fp16 form:
    alloc_workspace(..., packed_zeros=True))."""
    return _product("awq_gemm", x, qweight, scales, zeros, workspace, out, group_size, _flags(False, silu_mul))


def awq_linear(x, qweight, scales, zeros, workspace=None, out=None, group_size: int = GROUP_SIZE,
               weights_static: bool = False, silu_mul: bool = False):
    """The layer with the documented M threshold: awq_gemv for M <= 16, else awq_gemm.
    Either zero-point form; with packed zero points at M > 16 the workspace
    must come from alloc_workspace(..., packed_zeros=True)."""
    entry = "awq_gemv" if x.shape[0] <= GEMV_MAX_M else "awq_gemm"
    return _product(entry, x, qweight, scales, zeros, workspace, out, group_size,
                    _flags(weights_static, silu_mul))


def awq_interleave_gate_up(qweight_gate, scales_gate, zeros_gate, qweight_up, scales_up, zeros_up,
                           group_size: int = GROUP_SIZE):
    """The fused gate/up weight layout (AWQ_FLAG_SILU_MUL) from two packed
    projections of N rows each: (qweight [2N, K/8], scales [G, 2N], zeros or
    None), 16-row tiles alternating gate, up. Device-side copies only."""
    _need(qweight_gate, "qweight_gate", torch.int32, 2)
    _need(qweight_up, "qweight_up", torch.int32, 2)
    _need(scales_gate, "scales_gate", torch.float16, 2)
    _need(scales_up, "scales_up", torch.float16, 2)
    zp = zeros_gate is not None
    if zp != (zeros_up is not None):
        raise ValueError("gate and up must both have zero points or both not")
    if qweight_gate.shape != qweight_up.shape or scales_gate.shape != scales_up.shape:
        raise ValueError("gate and up must have the same shapes")
    N, K = qweight_gate.shape[0], qweight_gate.shape[1] * 8
    dev = qweight_gate.device
    q = torch.empty((2 * N, K // 8), dtype=torch.int32, device=dev)
    s = torch.empty((scales_gate.shape[0], 2 * N), dtype=torch.float16, device=dev)
    z = torch.empty_like(s) if zp else None
    with torch.cuda.device(dev):
        _check("awq_interleave_gate_up", lib().awq_interleave_gate_up(
            _ptr(qweight_gate), _ptr(scales_gate), _ptr(zeros_gate), _ptr(qweight_up), _ptr(scales_up),
            _ptr(zeros_up), N, K, _cfg(zp, group_size), _ptr(q), _ptr(s), _ptr(z), _stream(dev)))
    return q, s, z


def awq_device_error(device=None) -> int:
    """Read and clear the device error word (bit 0: a bounded wait in awq_gemm gave up)."""
    v = ctypes.c_uint32(0)
    dev = device if device is not None else torch.cuda.current_device()
    with torch.cuda.device(dev):
        _check("awq_device_error", lib().awq_device_error(ctypes.byref(v), _stream(dev)))
    return int(v.value)


def awq_concat_rows(parts, group_size: int = GROUP_SIZE):
    """Concatenate packed projections [(qweight, scales, zeros or None), ...]
    sharing K along N (q, k and v into one layer): returns (qweight
    [sum N, K/8], scales [G, sum N], zeros or None). Device-side copies only."""
    parts = list(parts)
    if not parts:
        raise ValueError("no parts")
    zp = parts[0][2] is not None
    K = parts[0][0].shape[1] * 8
    for q, s, z in parts:
        _need(q, "qweight", torch.int32, 2)
        _need(s, "scales", torch.float16, 2)
        if (z is not None) != zp:
            raise ValueError("all parts must have zero points or none")
        if q.shape[1] * 8 != K:
            raise ValueError("all parts must share K")
    n = len(parts)
    Ns = (_I64 * n)(*[q.shape[0] for q, _, _ in parts])
    qs = (_P * n)(*[q.data_ptr() for q, _, _ in parts])
    ss = (_P * n)(*[s.data_ptr() for _, s, _ in parts])
    zs = (_P * n)(*[(z.data_ptr() if z is not None else None) for _, _, z in parts])
    total = sum(Ns)
    dev = parts[0][0].device
    q = torch.empty((total, K // 8), dtype=torch.int32, device=dev)
    s = torch.empty((parts[0][1].shape[0], total), dtype=torch.float16, device=dev)
    z = torch.empty_like(s) if zp else None
    with torch.cuda.device(dev):
        _check("awq_concat_rows", lib().awq_concat_rows(n, qs, ss, zs, Ns, K, _cfg(zp, group_size),
                                                        _ptr(q), _ptr(s), _ptr(z), _stream(dev)))
    return q, s, z


def awq_search_scale(W: torch.Tensor, X: torch.Tensor, zero_point: bool = True, n_grid: int = 20,
                     duo: bool = True, group_size: int = GROUP_SIZE):
    """Activation-aware scale search for the layer W [N, K] on calibration
    inputs X [Ms, K]: returns (scales fp32 [K] of the lowest-error grid point,
    losses fp32 [n_grid]). All on the device (see awq.h)."""
    _need(W, "W", torch.float16, 2)
    _need(X, "X", torch.float16, 2)
    N, K = W.shape
    Ms = X.shape[0]
    if X.shape[1] != K:
        raise ValueError("X must be [Ms, K] for W [N, K]")
    _same_device(W, X=X)
    cfg = _cfg(zero_point, group_size)
    n = ctypes.c_size_t(0)
    with torch.cuda.device(W.device):
        _check("awq_search_scale_workspace_bytes",
               lib().awq_search_scale_workspace_bytes(N, K, Ms, cfg, ctypes.byref(n)))
        ws = torch.empty(n.value, dtype=torch.uint8, device=W.device)
        scales = torch.empty(K, dtype=torch.float32, device=W.device)
        losses = torch.empty(n_grid, dtype=torch.float32, device=W.device)
        _check("awq_search_scale", lib().awq_search_scale(
            _ptr(W), N, K, _ptr(X), Ms, cfg, n_grid, 1 if duo else 0, _ptr(scales), _ptr(losses), _ptr(ws),
            n.value, _stream(W.device)))
    return scales, losses


def awq_apply_scale(W: torch.Tensor, scales: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """fp16(W[n, k] * s[k]): the weights of a layer whose input is divided by s."""
    _need(W, "W", torch.float16, 2)
    _need(scales, "scales", torch.float32, 1)
    N, K = W.shape
    if scales.shape[0] != K:
        raise ValueError("scales must be [K]")
    if out is None:
        out = torch.empty_like(W)
    _need(out, "out", torch.float16, 2)
    _out_shape(out, (N, K))
    _same_device(W, scales=scales, out=out)
    with torch.cuda.device(W.device):
        _check("awq_apply_scale", lib().awq_apply_scale(_ptr(W), _ptr(scales), N, K, _ptr(out), _stream(W.device)))
    return out


def awq_search_clip(W: torch.Tensor, X: torch.Tensor, zero_point: bool = True, n_grid: int = 20,
                    max_shrink: float = 0.5, group_size: int = GROUP_SIZE) -> torch.Tensor:
    """Clipping-ratio search for W [N, K] on calibration inputs X [Ms, K]:
    returns the ratios fp32 [K/group_size, N] (see awq.h)."""
    _need(W, "W", torch.float16, 2)
    _need(X, "X", torch.float16, 2)
    N, K = W.shape
    if X.shape[1] != K:
        raise ValueError("X must be [Ms, K] for W [N, K]")
    _same_device(W, X=X)
    n = ctypes.c_size_t(0)
    with torch.cuda.device(W.device):
        _check("awq_search_clip_workspace_bytes", lib().awq_search_clip_workspace_bytes(K, ctypes.byref(n)))
        ws = torch.empty(n.value, dtype=torch.uint8, device=W.device)
        ratios = torch.empty((K // group_size, N), dtype=torch.float32, device=W.device)
        _check("awq_search_clip", lib().awq_search_clip(
            _ptr(W), N, K, _ptr(X), X.shape[0], _cfg(zero_point, group_size), n_grid, float(max_shrink),
            _ptr(ratios), _ptr(ws), n.value, _stream(W.device)))
    return ratios


def awq_apply_clip(W: torch.Tensor, ratios: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """W with each (row, group) clipped to ratio * max|w| of the group (fp16)."""
    _need(W, "W", torch.float16, 2)
    _need(ratios, "ratios", torch.float32, 2)
    N, K = W.shape
    if ratios.shape != (K // GROUP_SIZE, N):
        raise ValueError("ratios must be [K/128, N]")
    if out is None:
        out = torch.empty_like(W)
    _need(out, "out", torch.float16, 2)
    _out_shape(out, (N, K))
    _same_device(W, ratios=ratios, out=out)
    with torch.cuda.device(W.device):
        _check("awq_apply_clip", lib().awq_apply_clip(_ptr(W), _ptr(ratios), N, K, _ptr(out), _stream(W.device)))
    return out


class GemvChain:
    """A prepared awq_gemv_chain call: several decode products in one launch,
    where a layer's input may be an earlier layer's output.

    layers: a list of dicts with keys
      qweight, scales, zeros  the packed layer (zeros None: symmetric; int32:
                              packed zero points, the same form for every layer)
      x                       fp16 [M, K] input, or None when x_from >= 0
      x_from                  -1 (default), or the index of the earlier layer
                              whose output is this layer's input
      silu_mul                fused gate/up layout (output N/2 columns)
      out                     optional fp16 output tensor
    The outputs (self.outputs) and a zero-filled workspace are allocated here
    (workspace: a uint8 device tensor to use instead; it must be zero-filled
    before the first call of this chain and then serve no other chain, or be
    zero-filled again in between); calling the object enqueues the launch on
    the current stream. The layer descriptors are built once, so repeated
    calls cost one library call.
    weights_static: no work still running on the stream writes the weights,
    so the launch may start streaming them before the previous kernel on the
    stream has finished."""

    def __init__(self, M: int, layers, weights_static: bool = False, device=None, workspace=None):
        layers = list(layers)
        n = len(layers)
        if not 1 <= n <= CHAIN_MAX_LAYERS:
            raise ValueError(f"a chain has 1 .. {CHAIN_MAX_LAYERS} layers")
        self.M = int(M)
        self.outputs = []
        self._keep = []
        arr = (GemvLayer * n)()
        dev = None
        for l, d in enumerate(layers):
            q, sc, z = d["qweight"], d["scales"], d.get("zeros")
            x_from = int(d.get("x_from", -1))
            silu = bool(d.get("silu_mul", False))
            if x_from >= 0:
                if not 0 <= x_from < l:
                    raise ValueError(f"layer {l}: x_from must name an earlier layer")
                x = self.outputs[x_from]
            else:
                x = d["x"]
            _need(x, f"layers[{l}].x", torch.float16, 2)
            if x.shape[0] != self.M:
                raise ValueError(f"layer {l}: x has {x.shape[0]} rows, the chain M = {self.M}")
            flags = (FLAG_WEIGHTS_STATIC if weights_static else 0) | (FLAG_SILU_MUL if silu else 0)
            _, N, K, flags = validate_product(x, q, sc, z, d.get("out"), None, GROUP_SIZE, flags)
            if dev is None:
                dev = x.device
            elif x.device != dev:
                raise ValueError(f"layer {l} is on {x.device}, the chain on {dev}")
            out = d.get("out")
            if out is None:
                out = torch.empty((self.M, N // 2 if silu else N), dtype=torch.float16, device=x.device)
            self.outputs.append(out)
            self._keep += [x, q, sc, z, out]
            arr[l] = GemvLayer(x.data_ptr(), q.data_ptr(), sc.data_ptr(), _ptr(z), out.data_ptr(), N, K,
                               _cfg(z is not None, GROUP_SIZE, flags), x_from)
        self.device = dev if device is None else torch.device(device)
        self._arr, self._n = arr, n
        nbytes = ctypes.c_size_t(0)
        with torch.cuda.device(self.device):
            _check("awq_gemv_chain_workspace_bytes",
                   lib().awq_gemv_chain_workspace_bytes(arr, n, self.M, ctypes.byref(nbytes)))
        if workspace is None:
            workspace = torch.zeros(max(int(nbytes.value), 16), dtype=torch.uint8, device=self.device)
        else:
            _need(workspace, "workspace", torch.uint8, 1)
            if workspace.device != self.device:
                raise ValueError(f"workspace is on {workspace.device}, the chain on {self.device}")
            if workspace.numel() < int(nbytes.value):
                raise ValueError(f"workspace has {workspace.numel()} bytes, the chain needs {int(nbytes.value)}")
        self.workspace = workspace
        self._ws = (self.workspace.data_ptr(), self.workspace.numel())

    def __call__(self):
        if self.device.index == torch.cuda.current_device():
            st = lib().awq_gemv_chain(self._arr, self._n, self.M, self._ws[0], self._ws[1],
                                      torch.cuda.current_stream().cuda_stream)
        else:
            with torch.cuda.device(self.device):
                st = lib().awq_gemv_chain(self._arr, self._n, self.M, self._ws[0], self._ws[1],
                                          torch.cuda.current_stream(self.device).cuda_stream)
        _check("awq_gemv_chain", st)
        return self.outputs


def awq_gemv_chain(M: int, layers, weights_static: bool = False):
    """One awq_gemv_chain call (see GemvChain); returns the layers' outputs."""
    return GemvChain(M, layers, weights_static)()


def awq_debug_set_wait_limit_ns(ns: int, device=None):
    """Test hook: the time limit of awq_gemv_chain's pipeline waits (0: the
    default 2 s). Synchronizes the device's current stream."""
    dev = device if device is not None else torch.cuda.current_device()
    with torch.cuda.device(dev):
        _check("awq_debug_set_wait_limit_ns", lib().awq_debug_set_wait_limit_ns(int(ns), _stream(dev)))
