"""The C ABI library on the host (no GPU): it loads, exports every symbol the
header declares, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

import w8_quantized_linear_b200 as bn
from w8_quantized_linear_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitnest.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return bn.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bitnest_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("bitnest_pack_planes", "bitnest_quantize_act", "bitnest_linear",
                     "bitnest_debug_group_sums", "bitnest_status_string"):
        assert required in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_status_strings(L):
    assert bn.status_string(0) == "ok"
    for s in range(1, 5):
        assert bn.status_string(s) not in ("ok", "unknown status")
    assert bn.status_string(99) == "unknown status"
    assert L.bitnest_version() >= 100


def test_select_path():
    assert bn.select_path(bn.DRAFT, 1, 4096, 4096) == bn.PATH_GEMV
    assert bn.select_path(bn.TARGET, 4, 14336, 4096) == bn.PATH_GEMV
    assert bn.select_path(bn.TARGET, 8, 4096, 14336) == bn.PATH_GEMV
    assert bn.select_path(bn.TARGET, 9, 4096, 4096) == bn.PATH_GEMV  # two token blocks
    assert bn.select_path(bn.TARGET, 16, 14336, 4096) == bn.PATH_GEMV
    assert bn.select_path(bn.TARGET, 17, 4096, 4096) == bn.PATH_TC
    assert bn.select_path(bn.TARGET, 9, 4096, 14336) == bn.PATH_TC  # codes too large to stage
    assert bn.select_path(bn.TARGET, 2048, 4096, 4096) == bn.PATH_TC


A = 0x10000  # fake, aligned, never dereferenced (every call below fails before a launch)
MIS = 0x10001


def _lin(L, mode=1, hi=A, lo=A, scale=A, xq=A, xs=A, xsum=A, M=4, N=64, K=128, y=A, g=0,
         bias=None, path=0):
    v = ctypes.c_void_p
    return L.bitnest_linear_path(mode, v(hi), v(lo), v(scale), v(xq), v(xs), v(xsum), M, N, K,
                                 v(y), g, v(bias) if bias else None, path, None)


def test_linear_argument_checks(L):
    assert _lin(L, mode=2) == 1
    assert _lin(L, g=64) == 1
    assert _lin(L, path=3) == 1
    assert _lin(L, K=0) == 2
    assert _lin(L, K=100) == 2
    assert _lin(L, K=4096 + 64) == 2
    assert _lin(L, M=-1) == 2
    assert _lin(L, hi=0) == 1
    assert _lin(L, scale=0) == 1
    # xsum is optional (the kernels form the group sums): a NULL xsum passes
    # the checks, as the misaligned output shows (nothing is launched)
    assert _lin(L, xsum=0, y=MIS) == 3
    assert _lin(L, xsum=0, M=0) == 0
    assert _lin(L, xsum=MIS) == 3
    assert _lin(L, y=0) == 1
    assert _lin(L, mode=1, lo=0) == 1
    assert _lin(L, mode=1, lo=MIS) == 3
    assert _lin(L, hi=MIS) == 3
    assert _lin(L, y=MIS) == 3
    assert _lin(L, bias=MIS) == 3
    # draft ignores lo entirely (NULL or misaligned)
    assert _lin(L, mode=0, lo=0, M=0) == 0
    assert _lin(L, mode=0, lo=MIS, M=0) == 0
    # empty problems launch nothing and succeed
    assert _lin(L, M=0) == 0
    assert _lin(L, N=0) == 0
    # an explicit GEMV path cannot take more than 8 tokens (checked before launch)
    assert _lin(L, M=9, path=1) == 2
    assert L.bitnest_device_wait_timeout is not None


def test_quantize_linear_argument_checks(L):
    v = ctypes.c_void_p

    def q(x=A, xq=A, xs=A, xsum=A, M=4, N=64, K=128, mode=1, g=0, path=0):
        return L.bitnest_quantize_linear(mode, v(A), v(A), v(A), v(x) if x else None, M, N, K,
                                         v(A), g, None, v(xq) if xq else None,
                                         v(xs) if xs else None, v(xsum) if xsum else None,
                                         path, None)

    assert q(x=0) == 1
    assert q(x=MIS) == 3
    assert q(xq=0) == 1
    assert q(xsum=MIS) == 3
    assert q(xsum=0, x=MIS) == 3  # a NULL xsum passes the checks (nothing launched)
    assert q(K=200) == 2
    assert q(g=7) == 1
    assert q(path=5) == 1
    assert q(M=9, path=1) == 2  # GEMV takes at most 8 tokens: nothing launched
    assert q(M=0) == 0
    assert q(N=0) == 0


def test_quantize_pack_sum_argument_checks(L):
    v = ctypes.c_void_p
    assert L.bitnest_quantize_act(v(A), 4, 128, 3, v(A), v(A), None, None) == 1
    assert L.bitnest_quantize_act(v(A), 4, 130, 0, v(A), v(A), None, None) == 2
    assert L.bitnest_quantize_act(None, 4, 128, 0, v(A), v(A), None, None) == 1
    assert L.bitnest_quantize_act(v(A), 4, 128, 0, v(MIS), v(A), None, None) == 3
    assert L.bitnest_quantize_act(v(A), 4, 128, 0, v(A), v(A), v(MIS), None) == 3
    assert L.bitnest_quantize_act(v(A), 0, 128, 0, v(A), v(A), None, None) == 0
    assert L.bitnest_pack_planes(v(A), None, 4, 127, v(A), None, None) == 2
    assert L.bitnest_pack_planes(None, None, 4, 128, v(A), None, None) == 1
    assert L.bitnest_pack_planes(v(A), v(A), 4, 128, v(A), None, None) == 1
    assert L.bitnest_pack_planes(v(A), None, 0, 128, v(A), None, None) == 0
    assert L.bitnest_act_group_sums(v(A), 4, 256, None, None) == 1
    assert L.bitnest_act_group_sums(v(A), 0, 256, v(A), None) == 0
    assert L.bitnest_debug_group_sums(1, v(A), None, v(A), v(A), 1, 1, 128, v(A), 0, None) == 1
    # debug sums without xsum: the checks pass it (misaligned S shows where they stop)
    assert L.bitnest_debug_group_sums(1, v(A), v(A), v(A), None, 1, 1, 128, v(MIS), 0, None) == 3
    assert L.bitnest_debug_group_sums(0, v(A), None, v(A), v(A), 0, 1, 128, v(A), 0, None) == 0


def test_python_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(bn, "_lib", None)
    monkeypatch.setattr(bn, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        bn.lib()


def test_linear_ws_argument_checks(L):
    """Split-K scratch: its size query and the checks on it (no launch)."""
    v = ctypes.c_void_p
    need = L.bitnest_linear_ws_bytes(1, 16, 300, 1024, 2)
    assert need > 0  # 3 weight tiles: the tensor-core path splits K
    assert L.bitnest_linear_ws_bytes(1, 2048, 4096, 4096, 2) == 0  # enough tiles
    assert L.bitnest_linear_ws_bytes(1, 1, 4096, 4096, 1) == 0  # the GEMV takes none
    assert L.bitnest_linear_ws_bytes(3, 16, 300, 1024, 2) == -1
    assert L.bitnest_linear_ws_bytes(1, 16, 300, 1000, 2) == -2
    assert L.bitnest_linear_ws_bytes(1, 0, 300, 1024, 2) == 0
    # automatic choice with scratch: the TMA-ring GEMV for 4 tokens; for 8
    # tokens at K = 14336 (too many to stage for it) the split tensor-core path
    assert L.bitnest_linear_ws_bytes(1, 4, 4096, 14336, 0) == 0
    assert L.bitnest_linear_ws_bytes(1, 8, 4096, 14336, 0) > 0
    assert bn.select_path(bn.TARGET, 8, 4096, 14336) == bn.PATH_GEMV  # without scratch

    def call(ws=A, nbytes=need, M=16, N=300, K=1024, path=2):
        return L.bitnest_linear_ws(1, v(A), v(A), v(A), v(A), v(A), v(A), M, N, K, v(A), 0,
                                   None, path, v(ws) if ws else None, nbytes, None)

    assert call(ws=0) == 1
    assert call(nbytes=need - 16) == 1
    assert call(ws=MIS) == 3
    assert call(K=200) == 2
    assert call(path=7) == 1
    assert call(M=0) == 0


def test_pack_weights_argument_checks(L):
    v = ctypes.c_void_p
    assert L.bitnest_pack_weights(v(A), 4, 200, v(A), v(A), v(A), None) == 2
    assert L.bitnest_pack_weights(None, 4, 128, v(A), v(A), v(A), None) == 1
    assert L.bitnest_pack_weights(v(A), 4, 128, v(A), None, v(A), None) == 1
    assert L.bitnest_pack_weights(v(A), 4, 128, v(A), v(A), v(MIS), None) == 3
    assert L.bitnest_pack_weights(v(A), 0, 128, None, None, None, None) == 0


def test_hadamard_quantize_argument_checks(L):
    v = ctypes.c_void_p
    assert L.bitnest_hadamard_quantize_act(v(A), 2, 1000, v(A), v(A), None, None) == 2
    assert L.bitnest_hadamard_quantize_act(v(A), 2, 384, v(A), v(A), None, None) == 2  # not p, 28p
    assert L.bitnest_hadamard_quantize_act(v(A), 2, 65536, v(A), v(A), None, None) == 2  # too long
    assert L.bitnest_hadamard_quantize_act(None, 2, 14336, v(A), v(A), None, None) == 1
    assert L.bitnest_hadamard_quantize_act(v(A), 2, 14336, v(MIS), v(A), None, None) == 3
    assert L.bitnest_hadamard_quantize_act(v(A), 0, 14336, None, None, None, None) == 0


def test_nested_attention_argument_checks(L):
    v = ctypes.c_void_p

    def call(mode=1, H=32, Hkv=8, D=128, T=10, lo=A, q=A, out=A):
        return L.bitnest_nested_attention(mode, v(q) if q else None, H, Hkv, D, T, v(A),
                                          v(lo) if lo else None, v(A), v(A),
                                          v(lo) if lo else None, v(A), v(out) if out else None,
                                          None)

    assert call(mode=2) == 1
    assert call(D=64) == 2
    assert call(H=24, Hkv=8) == 2  # 3 query heads per KV head
    assert call(H=30, Hkv=8) == 2
    assert call(T=0) == 2
    assert call(q=0) == 1
    assert call(lo=0) == 1  # the target needs the lo planes
    assert call(out=MIS) == 3
