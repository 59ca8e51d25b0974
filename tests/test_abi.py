"""C ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before any CUDA call.

Every call below fails validation before the library touches the CUDA
runtime (null pointers, bad sizes, bad configuration, misalignment), so the
pointers passed are never dereferenced."""

import ctypes
import os
import re

import pytest
import torch

import weight_only_int4_gemv_b200 as awq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "awq.h")

OK, NULL, SHAPE, ALIGN, UNSUP, CUDA, WS = range(7)
A = 0x10000          # a 16-byte aligned fake address (never dereferenced)
MIS = 0x10002        # a misaligned fake address


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"AWQ_API\s+[\w\s\*]+?\b(awq_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(awq.LIB_PATH):
        from weight_only_int4_gemv_b200 import build
        build.build()
    return awq.lib()


def cfg(g=128, zp=1, flags=0):
    return awq.QConfig(g, zp, flags)


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for s in ["awq_pseudo_quantize_pack", "awq_dequant", "awq_gemv", "awq_gemm",
              "awq_workspace_bytes", "awq_status_string", "awq_abi_version", "awq_device_error",
              "awq_interleave_gate_up", "awq_concat_rows", "awq_search_scale",
              "awq_search_scale_workspace_bytes", "awq_apply_scale", "awq_search_clip",
              "awq_search_clip_workspace_bytes", "awq_apply_clip", "awq_pack_zeros", "awq_unpack_zeros"]:
        assert s in syms


def test_library_exports_every_declared_symbol(L):
    for s in declared_symbols():
        assert hasattr(L, s), s
        assert ctypes.cast(getattr(L, s), ctypes.c_void_p).value


def test_abi_version_matches_header(L):
    m = re.search(r"#define AWQ_ABI_VERSION (\d+)", open(HEADER).read())
    assert L.awq_abi_version() == int(m.group(1))


def test_status_strings(L):
    for st in range(7):
        assert L.awq_status_string(st)
    assert L.awq_status_string(99) == b"unknown status"


def _gemv(L, x=A, q=A, s=A, z=A, M=1, N=64, K=256, c=None, y=A, entry="awq_gemv"):
    fn = getattr(L, entry)
    return fn(ctypes.c_void_p(x), ctypes.c_void_p(q), ctypes.c_void_p(s),
              ctypes.c_void_p(z) if z else None, M, N, K, c or cfg(), ctypes.c_void_p(y),
              None, 0, None)


@pytest.mark.parametrize("entry", ["awq_gemv", "awq_gemm"])
def test_product_validation(L, entry):
    assert _gemv(L, c=cfg(g=64), entry=entry) == UNSUP          # only g = 128 is built
    assert _gemv(L, c=cfg(zp=2), entry=entry) == UNSUP
    assert _gemv(L, K=200, entry=entry) == SHAPE                # K % 128 != 0
    assert _gemv(L, K=0, entry=entry) == SHAPE
    assert _gemv(L, N=-1, entry=entry) == SHAPE
    assert _gemv(L, x=0, entry=entry) == NULL
    assert _gemv(L, q=0, entry=entry) == NULL
    assert _gemv(L, y=0, entry=entry) == NULL
    assert _gemv(L, z=0, entry=entry) == NULL                   # asym needs zeros
    assert _gemv(L, z=A, c=cfg(zp=0), entry=entry) == SHAPE     # sym takes no zeros
    assert _gemv(L, x=MIS, entry=entry) == ALIGN
    assert _gemv(L, y=MIS, entry=entry) == ALIGN
    assert _gemv(L, N=0, entry=entry) == OK                     # empty: no work, no CUDA call
    assert _gemv(L, c=cfg(flags=8), entry=entry) == UNSUP       # undefined flag bits
    assert _gemv(L, c=cfg(flags=0x80000000), entry=entry) == UNSUP
    assert _gemv(L, N=0, c=cfg(flags=awq.FLAG_WEIGHTS_STATIC), entry=entry) == OK
    # the fused gate/up layout needs whole 32-row tile pairs
    assert _gemv(L, N=48, c=cfg(flags=awq.FLAG_SILU_MUL), entry=entry) == SHAPE
    assert _gemv(L, N=0, c=cfg(flags=awq.FLAG_SILU_MUL), entry=entry) == OK


def test_concat_rows_validation(L):
    f = L.awq_concat_rows
    P = ctypes.c_void_p
    ptrs = (P * 2)(A, A)
    Ns = (ctypes.c_int64 * 2)(16, 32)
    # every case below is rejected before any CUDA call (the pointers are fake)
    assert f(0, ptrs, ptrs, ptrs, Ns, 256, cfg(), P(A), P(A), P(A), None) == SHAPE       # no parts
    assert f(17, ptrs, ptrs, ptrs, Ns, 256, cfg(), P(A), P(A), P(A), None) == SHAPE      # too many
    assert f(2, ptrs, ptrs, ptrs, Ns, 200, cfg(), P(A), P(A), P(A), None) == SHAPE       # K % 128
    assert f(2, None, ptrs, ptrs, Ns, 256, cfg(), P(A), P(A), P(A), None) == NULL
    assert f(2, ptrs, ptrs, None, Ns, 256, cfg(), P(A), P(A), P(A), None) == NULL        # asym needs zeros
    assert f(2, ptrs, ptrs, ptrs, Ns, 256, cfg(), P(A), P(A), None, None) == NULL        # zeros out
    assert f(2, ptrs, ptrs, ptrs, Ns, 256, cfg(zp=0), P(A), P(A), None, None) == SHAPE   # sym: no zeros
    assert f(2, ptrs, ptrs, ptrs, Ns, 256, cfg(flags=4), P(A), P(A), P(A), None) == UNSUP
    zero = (ctypes.c_int64 * 2)(0, 0)
    assert f(2, ptrs, ptrs, ptrs, zero, 256, cfg(), P(A), P(A), P(A), None) == OK       # empty
    neg = (ctypes.c_int64 * 2)(16, -1)
    assert f(2, ptrs, ptrs, ptrs, neg, 256, cfg(), P(A), P(A), P(A), None) == SHAPE


def test_search_scale_validation(L):
    P = ctypes.c_void_p
    n = ctypes.c_size_t(0)
    ws = L.awq_search_scale_workspace_bytes
    assert ws(64, 256, 8, cfg(), None) == NULL
    assert ws(60, 256, 8, cfg(), ctypes.byref(n)) == SHAPE          # N % 8
    assert ws(64, 200, 8, cfg(), ctypes.byref(n)) == SHAPE          # K % 128
    assert ws(64, 256, 0, cfg(), ctypes.byref(n)) == SHAPE          # no calibration rows
    assert ws(64, 256, 8, cfg(flags=1), ctypes.byref(n)) == UNSUP    # no flags
    # the size depends on the device's SM count: without a GPU the query reports CUDA
    st = ws(64, 256, 8, cfg(), ctypes.byref(n))
    assert st in (OK, CUDA) and (st == CUDA or n.value > 0)
    f = L.awq_search_scale
    big = 1 << 30
    # every case below is rejected before any CUDA call (the pointers are fake)
    assert f(P(A), 64, 256, P(A), 8, cfg(), 0, 1, P(A), P(A), P(A), big, None) == SHAPE      # n_grid
    assert f(P(A), 64, 256, P(A), 8, cfg(), 65, 1, P(A), P(A), P(A), big, None) == SHAPE
    assert f(None, 64, 256, P(A), 8, cfg(), 10, 1, P(A), P(A), P(A), big, None) == NULL
    assert f(P(A), 64, 256, P(A), 8, cfg(), 10, 1, P(A), P(A), None, big, None) == NULL
    assert f(P(MIS), 64, 256, P(A), 8, cfg(), 10, 1, P(A), P(A), P(A), big, None) == ALIGN
    if st == OK:   # (on a GPU machine) a workspace one short of the need is refused before any launch
        assert f(P(A), 64, 256, P(A), 8, cfg(), 10, 1, P(A), P(A), P(A), n.value - 16, None) == WS
    ap = L.awq_apply_scale
    assert ap(P(A), P(A), 0, 256, P(A), None) == OK
    assert ap(None, P(A), 8, 256, P(A), None) == NULL
    assert ap(P(A), P(A), -1, 256, P(A), None) == SHAPE


def test_search_clip_validation(L):
    P = ctypes.c_void_p
    n = ctypes.c_size_t(0)
    assert L.awq_search_clip_workspace_bytes(200, ctypes.byref(n)) == SHAPE
    assert L.awq_search_clip_workspace_bytes(256, ctypes.byref(n)) == OK and n.value == 2 * 128 * 128 * 4
    f = L.awq_search_clip
    big = 1 << 30
    # every case below is rejected before any CUDA call (the pointers are fake)
    assert f(P(A), 64, 256, P(A), 8, cfg(), 0, ctypes.c_float(0.5), P(A), P(A), big, None) == SHAPE
    assert f(P(A), 64, 256, P(A), 8, cfg(), 10, ctypes.c_float(1.0), P(A), P(A), big, None) == SHAPE
    assert f(P(A), 64, 256, P(A), 8, cfg(), 10, ctypes.c_float(-0.1), P(A), P(A), big, None) == SHAPE
    assert f(P(A), 60, 256, P(A), 8, cfg(), 10, ctypes.c_float(0.5), P(A), P(A), big, None) == SHAPE
    assert f(None, 64, 256, P(A), 8, cfg(), 10, ctypes.c_float(0.5), P(A), P(A), big, None) == NULL
    assert f(P(A), 64, 256, P(A), 8, cfg(), 10, ctypes.c_float(0.5), P(A), P(A), n.value - 4, None) == WS
    assert f(P(A), 64, 256, P(A), 8, cfg(flags=2), 10, ctypes.c_float(0.5), P(A), P(A), big, None) == UNSUP
    ap = L.awq_apply_clip
    assert ap(P(A), P(A), 0, 256, P(A), None) == OK
    assert ap(P(A), P(A), 8, 200, P(A), None) == SHAPE
    assert ap(P(MIS), P(A), 8, 256, P(A), None) == ALIGN


def test_interleave_gate_up_validation(L):
    f = L.awq_interleave_gate_up
    P = ctypes.c_void_p
    ok6 = [P(A)] * 6
    # every case below is rejected before any CUDA call (the pointers are fake)
    assert f(*ok6, 24, 256, cfg(), P(A), P(A), P(A), None) == SHAPE        # N % 16
    assert f(*ok6, 32, 200, cfg(), P(A), P(A), P(A), None) == SHAPE        # K % 128
    assert f(*ok6, 0, 256, cfg(), P(A), P(A), P(A), None) == OK            # empty
    assert f(None, *ok6[1:], 32, 256, cfg(), P(A), P(A), P(A), None) == NULL
    assert f(*ok6, 32, 256, cfg(), P(A), P(A), None, None) == NULL           # asym: zeros out
    assert f(*ok6, 32, 256, cfg(zp=0), P(A), P(A), None, None) == SHAPE      # sym takes no zeros
    assert f(*ok6, 32, 256, cfg(flags=4), P(A), P(A), P(A), None) == UNSUP


def test_gemv_batch_range(L):
    assert _gemv(L, M=0) == SHAPE
    assert _gemv(L, M=17) == SHAPE
    assert _gemv(L, M=0, entry="awq_gemm") == OK                # empty batch
    assert _gemv(L, M=-3, entry="awq_gemm") == SHAPE


def test_quantize_and_dequant_validation(L):
    q = L.awq_pseudo_quantize_pack
    P = ctypes.c_void_p
    assert q(None, 8, 256, cfg(), P(A), P(A), P(A), None) == NULL
    assert q(P(A), 8, 256, cfg(), P(A), P(A), None, None) == NULL
    assert q(P(A), 8, 256, cfg(zp=0), P(A), P(A), P(A), None) == SHAPE
    assert q(P(A), 8, 100, cfg(), P(A), P(A), P(A), None) == SHAPE
    assert q(P(MIS), 8, 256, cfg(), P(A), P(A), P(A), None) == ALIGN
    assert q(P(A), 0, 256, cfg(), P(A), P(A), P(A), None) == OK
    assert q(P(A), 8, 256, cfg(flags=4), P(A), P(A), P(A), None) == UNSUP
    d = L.awq_dequant
    assert d(None, P(A), P(A), 8, 256, cfg(), P(A), None) == NULL
    assert d(P(A), P(A), P(A), 8, 256, cfg(g=32), P(A), None) == UNSUP
    assert d(P(A), P(A), P(A), 8, 256, cfg(), P(MIS), None) == ALIGN
    assert d(P(A), P(A), P(A), 0, 256, cfg(), P(A), None) == OK


def test_packed_zeros_validation(L):
    PZ = awq.FLAG_PACKED_ZEROS
    assert PZ == int(re.search(r"#define AWQ_FLAG_PACKED_ZEROS (\d+)u", open(HEADER).read()).group(1))
    P = ctypes.c_void_p
    # every case below is rejected (or has no work) before any CUDA call (the pointers are fake)
    for entry in ("awq_gemv", "awq_gemv_noalloc"):
        f = getattr(L, entry)
        args = lambda N, c, z=A: (P(A), P(A), P(A), P(z) if z else None, 1, N, 256, c, P(A))
        tail = (None, 0, None) if entry == "awq_gemv" else (None,)
        assert f(*args(64, cfg(zp=0, flags=PZ), z=0), *tail) == UNSUP     # packed zeros need zero_point = 1
        assert f(*args(48, cfg(flags=PZ)), *tail) == SHAPE                # N % 32
        assert f(*args(0, cfg(flags=PZ)), *tail) == OK                    # empty
        assert f(*args(64, cfg(flags=PZ), z=0), *tail) == NULL
        assert f(*args(64, cfg(flags=PZ), z=MIS), *tail) == ALIGN
    # the GEMM unpacks packed zero points into its workspace: none given, or too small
    assert _gemv(L, M=32, c=cfg(flags=PZ), entry="awq_gemm") == WS
    g = L.awq_gemm
    assert g(P(A), P(A), P(A), P(A), 32, 64, 256, cfg(flags=PZ), P(A), P(A), 255, None) == WS
    assert g(P(A), P(A), P(A), P(A), 32, 64, 256, cfg(flags=PZ), P(A), P(MIS), 256, None) == ALIGN
    assert _gemv(L, M=32, N=48, c=cfg(flags=PZ), entry="awq_gemm") == SHAPE   # N % 32
    assert _gemv(L, M=32, c=cfg(zp=0, flags=PZ), z=0, entry="awq_gemm") == UNSUP
    n = ctypes.c_size_t(7)
    # M > 16: the fp16 copy of the zero points, G x N x 2 bytes
    assert L.awq_workspace_bytes(32, 64, 256, cfg(flags=PZ), ctypes.byref(n)) == OK and n.value == 2 * 64 * 2
    assert L.awq_workspace_bytes(32, 64, 256, cfg(), ctypes.byref(n)) == OK and n.value == 0
    assert L.awq_workspace_bytes(1, 48, 256, cfg(flags=PZ), ctypes.byref(n)) == SHAPE
    assert L.awq_workspace_bytes(1, 0, 256, cfg(flags=PZ), ctypes.byref(n)) == OK and n.value == 0
    d = L.awq_dequant
    assert d(P(A), P(A), P(A), 12, 256, cfg(flags=PZ), P(A), None) == SHAPE     # N % 8
    assert d(P(A), P(A), None, 8, 256, cfg(zp=0, flags=PZ), P(A), None) == UNSUP
    assert d(P(A), P(A), P(MIS), 8, 256, cfg(flags=PZ), P(A), None) == ALIGN
    assert d(P(A), P(A), P(A), 0, 256, cfg(flags=PZ), P(A), None) == OK
    for f in (L.awq_pack_zeros, L.awq_unpack_zeros):
        assert f(P(A), 2, 12, P(A), None) == SHAPE       # N % 8
        assert f(P(A), -1, 16, P(A), None) == SHAPE
        assert f(P(A), 2, -8, P(A), None) == SHAPE
        assert f(P(A), 0, 16, P(A), None) == OK          # empty
        assert f(P(A), 2, 0, None, None) == OK
        assert f(None, 2, 16, P(A), None) == NULL
        assert f(P(A), 2, 16, None, None) == NULL
        assert f(P(MIS), 2, 16, P(A), None) == ALIGN
        assert f(P(A), 2, 16, P(MIS), None) == ALIGN
    # entry points that copy or write zero points take the fp16 form only
    assert L.awq_pseudo_quantize_pack(P(A), 8, 256, cfg(flags=PZ), P(A), P(A), P(A), None) == UNSUP


def test_binding_packed_zeros_shapes():
    with pytest.raises(ValueError):
        awq.awq_pack_zeros(torch.zeros(2, 16, dtype=torch.float16))     # not a CUDA tensor


def test_workspace_query_validation(L):
    n = ctypes.c_size_t(7)
    assert L.awq_workspace_bytes(1, 64, 256, cfg(), None) == NULL
    assert L.awq_workspace_bytes(1, 64, 250, cfg(), ctypes.byref(n)) == SHAPE
    assert L.awq_workspace_bytes(0, 64, 256, cfg(), ctypes.byref(n)) == OK and n.value == 0
    assert L.awq_workspace_bytes(4, 0, 256, cfg(), ctypes.byref(n)) == OK and n.value == 0


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 256, dtype=torch.float16)
    with pytest.raises(ValueError, match="CUDA"):
        awq.awq_gemv(x, torch.zeros(8, 32, dtype=torch.int32), torch.zeros(8, 2, dtype=torch.float16), None)


def _layer(M=2, N=64, K=256, device="cpu", packed=False):
    x = torch.zeros(M, K, dtype=torch.float16, device=device)
    q = torch.zeros(N, K // 8, dtype=torch.int32, device=device)
    s = torch.zeros(K // 128, N, dtype=torch.float16, device=device)
    z = (torch.zeros(K // 128, N // 8, dtype=torch.int32, device=device) if packed
         else torch.zeros(K // 128, N, dtype=torch.float16, device=device))
    return x, q, s, z


def test_binding_validation_accepts_a_consistent_layer():
    x, q, s, z = _layer()
    assert awq.validate_product(x, q, s, z) == (2, 64, 256, 0)
    assert awq.validate_product(x, q, s, None) == (2, 64, 256, 0)
    out = torch.zeros(2, 32, dtype=torch.float16)
    assert awq.validate_product(x, q, s, z, out, flags=awq.FLAG_SILU_MUL)[3] == awq.FLAG_SILU_MUL
    xp, qp, sp, zp = _layer(packed=True)
    assert awq.validate_product(xp, qp, sp, zp)[3] == awq.FLAG_PACKED_ZEROS


def test_binding_validation_rejects_wrong_out_shape():
    """An `out` smaller than [M, N] would be written past its end."""
    x, q, s, z = _layer()
    for shape in [(2, 32), (1, 64), (2, 65), (64, 2)]:
        with pytest.raises(ValueError, match="out must be"):
            awq.validate_product(x, q, s, z, torch.zeros(*shape, dtype=torch.float16))
    with pytest.raises(ValueError, match="out must be"):      # silu_mul: [M, N/2]
        awq.validate_product(x, q, s, z, torch.zeros(2, 64, dtype=torch.float16), flags=awq.FLAG_SILU_MUL)


def test_binding_validation_rejects_wrong_metadata_shapes():
    x, q, s, z = _layer()
    with pytest.raises(ValueError, match="scales"):
        awq.validate_product(x, q, torch.zeros(1, 64, dtype=torch.float16), z)     # undersized scales
    with pytest.raises(ValueError):
        awq.validate_product(x, q, s, torch.zeros(2, 32, dtype=torch.float16))      # undersized zeros
    with pytest.raises(ValueError):
        awq.validate_product(x, q, s, torch.zeros(2, 4, dtype=torch.int32))        # undersized qzeros
    with pytest.raises(ValueError, match="qweight"):
        awq.validate_product(x, torch.zeros(64, 16, dtype=torch.int32), s, z)


def test_binding_validation_rejects_operands_on_another_device():
    """Operands on different devices would make the kernel read another
    device's memory; the 'meta' device stands in for a second device here."""
    x, q, s, z = _layer()
    xm, qm, sm, zm = _layer(device="meta")
    out_m = torch.zeros(2, 64, dtype=torch.float16, device="meta")
    for args in [(x, qm, s, z), (x, q, sm, z), (x, q, s, zm)]:
        with pytest.raises(ValueError, match="device"):
            awq.validate_product(*args)
    with pytest.raises(ValueError, match="device"):
        awq.validate_product(x, q, s, z, out_m)
    with pytest.raises(ValueError, match="device"):
        awq.validate_product(x, q, s, z, workspace=torch.zeros(16, dtype=torch.uint8, device="meta"))


def test_noalloc_binding_runs_the_same_checks():
    """awq_gemv_noalloc goes through the same validation as awq_gemv: with a
    CUDA-less x it stops at the device check, and its shape checks are those
    of validate_product (exercised above)."""
    import inspect
    src = inspect.getsource(awq.awq_gemv_noalloc)
    assert "validate_product(" in src
    x, q, s, z = _layer()
    with pytest.raises(ValueError, match="CUDA"):
        awq.awq_gemv_noalloc(x, q, torch.zeros(1, 64, dtype=torch.float16), z)
