"""BitNest bit-nested W4/W8 quantised linear layer on B200 (sm_100a).

Thin Python binding over the C ABI of ``libbitnest.so`` (declared in
``include/bitnest.h``).  Every function here only marshals arguments: it
allocates outputs with torch, passes device pointers and the current CUDA
stream, and raises on a non-zero status.  All computation runs in the CUDA
kernels of the library; there is no CPU path.  If the library is missing the
first call raises.

One stored 8-bit weight code serves two models (BitNest-Llama-3-8B model
card, section "Files"): the draft (W4A8) reads the hi nibble plane only, the
target (W8A8) reads the hi and lo planes.
"""
from __future__ import annotations

import ctypes
import os

DRAFT = 0
TARGET = 1
PATH_AUTO = 0
PATH_GEMV = 1
PATH_TC = 2
PATH_OVERLAP = 0x100  # OR into path: stream the weights before the previous kernel ends
GEMV_MAX_M = 16
GROUP = 128

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitnest.so")

_lib = None


class BitnestError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """Load libbitnest.so (built in-tree by build.py); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m w8_quantized_linear_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    L.bitnest_status_string.argtypes = [I]
    L.bitnest_status_string.restype = ctypes.c_char_p
    L.bitnest_version.restype = I
    L.bitnest_device_wait_timeout.argtypes = [I]
    L.bitnest_device_wait_timeout.restype = I
    L.bitnest_pack_planes.argtypes = [P, P, I64, I64, P, P, P]
    L.bitnest_debug_wait_probe.argtypes = [P]
    L.bitnest_debug_wait_probe.restype = I
    L.bitnest_pack_weights.argtypes = [P, I64, I64, P, P, P, P]
    L.bitnest_hadamard_quantize_act.argtypes = [P, I64, I64, P, P, P, P]
    L.bitnest_nested_attention.argtypes = [I, P, I64, I64, I64, I64, P, P, P, P, P, P, P, P]
    L.bitnest_quantize_act.argtypes = [P, I64, I64, I, P, P, P, P]
    L.bitnest_act_group_sums.argtypes = [P, I64, I64, P, P]
    L.bitnest_linear.argtypes = [I, P, P, P, P, P, P, I64, I64, I64, P, I, P, P]
    L.bitnest_linear_path.argtypes = [I, P, P, P, P, P, P, I64, I64, I64, P, I, P, I, P]
    L.bitnest_select_path.argtypes = [I, I64, I64, I64]
    L.bitnest_debug_group_sums.argtypes = [I, P, P, P, P, I64, I64, I64, P, I, P]
    L.bitnest_quantize_linear.argtypes = [I, P, P, P, P, I64, I64, I64, P, I, P, P, P, P, I, P]
    L.bitnest_linear_ws.argtypes = [I, P, P, P, P, P, P, I64, I64, I64, P, I, P, I, P, I64, P]
    L.bitnest_linear_static_ws.argtypes = [I, P, P, P, P, P, P, I64, I64, I64, P, I, P, I, P]
    L.bitnest_linear_ws_bytes.argtypes = [I, I64, I64, I64, I]
    L.bitnest_linear_ws_bytes.restype = I64
    L.bitnest_spec_work_bytes.argtypes = [I64, I64, I]
    L.bitnest_spec_work_bytes.restype = I64
    L.bitnest_spec_rounds.argtypes = [P, I, I, P, I64, P, P, P, I64, P]
    L.bitnest_spec_greedy.argtypes = [P, I, P, I64, P, P, P, I64, P]
    for name in ("bitnest_pack_planes", "bitnest_pack_weights", "bitnest_quantize_act",
                 "bitnest_act_group_sums", "bitnest_hadamard_quantize_act",
                 "bitnest_nested_attention",
                 "bitnest_linear", "bitnest_linear_path", "bitnest_select_path",
                 "bitnest_debug_group_sums", "bitnest_quantize_linear", "bitnest_linear_ws",
                 "bitnest_linear_static_ws", "bitnest_spec_rounds", "bitnest_spec_greedy"):
        getattr(L, name).restype = I
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().bitnest_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != 0:
        raise BitnestError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t=None):
    import torch

    dev = t.device if t is not None else None
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def device_wait_timeout(reset: bool = False) -> int:
    """1 if a bounded in-kernel wait gave up since the last reset, else 0."""
    v = int(lib().bitnest_device_wait_timeout(1 if reset else 0))
    if v < 0:
        raise BitnestError(-v, "bitnest_device_wait_timeout")
    return v


def debug_wait_probe() -> None:
    """Test hook: a kernel whose bounded wait gives up and sets the flag that
    device_wait_timeout reports (clear it afterwards)."""
    _check(lib().bitnest_debug_wait_probe(_stream()), "bitnest_debug_wait_probe")


def select_path(mode: int, M: int, N: int, K: int) -> int:
    return int(lib().bitnest_select_path(int(mode), int(M), int(N), int(K)))


def pack_planes(uh, ul=None):
    """uint8 nibbles [N, K] (and optionally ul) -> planes uint8 [N, K/2]."""
    import torch

    N, K = uh.shape
    hi = torch.empty((N, K // 2), dtype=torch.uint8, device=uh.device)
    lo = torch.empty_like(hi) if ul is not None else None
    _check(lib().bitnest_pack_planes(_ptr(uh), _ptr(ul), N, K, _ptr(hi), _ptr(lo), _stream(uh)),
           "bitnest_pack_planes")
    return hi, lo


def pack_weights(w, out=None):
    """fp16 weights [N, K] -> (hi, lo uint8 [N, K/2], scale fp16 [N, K/128]):
    round-to-nearest 4-bit high nibble, closed-form residual low nibble."""
    import torch

    N, K = w.shape
    if out is None:
        out = (torch.empty((N, K // 2), dtype=torch.uint8, device=w.device),
               torch.empty((N, K // 2), dtype=torch.uint8, device=w.device),
               torch.empty((N, K // GROUP), dtype=torch.float16, device=w.device))
    hi, lo, sc = out
    _check(lib().bitnest_pack_weights(_ptr(w), N, K, _ptr(hi), _ptr(lo), _ptr(sc), _stream(w)),
           "bitnest_pack_weights")
    return hi, lo, sc


def quantize_act(x, act_group: int = 0, with_sum: bool = True, out=None):
    """fp16 [M, K] -> (xq int8 [M, K], xscale fp32 [M] or [M, K/128], xsum int32 [M, K/128])."""
    import torch

    M, K = x.shape
    if out is None:
        xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
        xs = torch.empty((M,) if act_group == 0 else (M, K // GROUP), dtype=torch.float32,
                         device=x.device)
        xsum = torch.empty((M, K // GROUP), dtype=torch.int32, device=x.device) if with_sum else None
    else:
        xq, xs, xsum = out
    _check(lib().bitnest_quantize_act(_ptr(x), M, K, int(act_group), _ptr(xq), _ptr(xs),
                                      _ptr(xsum), _stream(x)), "bitnest_quantize_act")
    return xq, xs, xsum


def hadamard_quantize_act(x, out=None):
    """down_proj input path: fp16 [M, K] -> rotated by x H / sqrt(K) and
    quantised per token: (xq int8 [M, K], xscale fp32 [M], xsum int32 [M, K/128])."""
    import torch

    M, K = x.shape
    if out is None:
        out = (torch.empty((M, K), dtype=torch.int8, device=x.device),
               torch.empty((M,), dtype=torch.float32, device=x.device),
               torch.empty((M, K // GROUP), dtype=torch.int32, device=x.device))
    xq, xs, xsum = out
    _check(lib().bitnest_hadamard_quantize_act(_ptr(x), M, K, _ptr(xq), _ptr(xs), _ptr(xsum),
                                               _stream(x)), "bitnest_hadamard_quantize_act")
    return xq, xs, xsum


def nested_attention(mode: int, q, k_planes, v_planes, Hkv: int, out=None):
    """Decode attention of one token over a nested KV cache: q fp16 [H, 128];
    k_planes / v_planes = pack_weights(rows [T * Hkv, 128]); fp32 [H, 128]."""
    import torch

    H, D = q.shape
    k_hi, k_lo, k_sc = k_planes
    v_hi, v_lo, v_sc = v_planes
    T = k_hi.shape[0] // Hkv
    o = out if out is not None else torch.empty((H, D), dtype=torch.float32, device=q.device)
    _check(lib().bitnest_nested_attention(int(mode), _ptr(q), H, int(Hkv), D, T, _ptr(k_hi),
                                          _ptr(k_lo), _ptr(k_sc), _ptr(v_hi), _ptr(v_lo),
                                          _ptr(v_sc), _ptr(o), _stream(q)),
           "bitnest_nested_attention")
    return o


def act_group_sums(xq, out=None):
    import torch

    M, K = xq.shape
    xsum = out if out is not None else torch.empty((M, K // GROUP), dtype=torch.int32,
                                                    device=xq.device)
    _check(lib().bitnest_act_group_sums(_ptr(xq), M, K, _ptr(xsum), _stream(xq)),
           "bitnest_act_group_sums")
    return xsum


def linear(mode: int, hi, lo, scale, xq, xscale, xsum, act_group: int = 0, bias=None,
           out=None, path: int = PATH_AUTO):
    """The nested linear layer: fp32 y [M, N]."""
    import torch

    M, K = xq.shape
    N = hi.shape[0]
    y = out if out is not None else torch.empty((M, N), dtype=torch.float32, device=xq.device)
    _check(lib().bitnest_linear_path(int(mode), _ptr(hi), _ptr(lo), _ptr(scale), _ptr(xq),
                                     _ptr(xscale), _ptr(xsum), M, N, K, _ptr(y), int(act_group),
                                     _ptr(bias), int(path), _stream(xq)), "bitnest_linear")
    return y


def linear_ws_bytes(mode: int, M: int, N: int, K: int, path: int = PATH_AUTO) -> int:
    """Scratch bytes `linear_ws` uses for this problem (0: no split of K)."""
    n = lib().bitnest_linear_ws_bytes(int(mode), int(M), int(N), int(K), int(path))
    if n < 0:
        _check(-n, "bitnest_linear_ws_bytes")
    return n


def workspace(nbytes: int, device):
    """Zeroed scratch for `linear_ws` (its counters must start at zero)."""
    import torch

    return torch.zeros(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def linear_ws(mode: int, hi, lo, scale, xq, xscale, xsum, ws, act_group: int = 0, bias=None,
              out=None, path: int = PATH_AUTO):
    """`linear` with scratch `ws` (from `workspace`) that lets the tensor-core
    path split K across CTAs when the layer has few output tiles."""
    import torch

    M, K = xq.shape
    N = hi.shape[0]
    y = out if out is not None else torch.empty((M, N), dtype=torch.float32, device=xq.device)
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().bitnest_linear_ws(int(mode), _ptr(hi), _ptr(lo), _ptr(scale), _ptr(xq),
                                   _ptr(xscale), _ptr(xsum), M, N, K, _ptr(y), int(act_group),
                                   _ptr(bias), int(path), _ptr(ws), nbytes, _stream(xq)),
           "bitnest_linear_ws")
    return y


def linear_static_ws(mode: int, hi, lo, scale, xq, xscale, xsum, act_group: int = 0,
                     bias=None, out=None, path: int = PATH_AUTO):
    """`linear_ws` on the library's own static device scratch (no allocation;
    calls that overlap in time race: see bitnest_linear_static_ws)."""
    import torch

    M, K = xq.shape
    N = hi.shape[0]
    y = out if out is not None else torch.empty((M, N), dtype=torch.float32, device=xq.device)
    _check(lib().bitnest_linear_static_ws(int(mode), _ptr(hi), _ptr(lo), _ptr(scale), _ptr(xq),
                                          _ptr(xscale), _ptr(xsum), M, N, K, _ptr(y),
                                          int(act_group), _ptr(bias), int(path), _stream(xq)),
           "bitnest_linear_static_ws")
    return y


def quantize_linear(mode: int, hi, lo, scale, x, act_group: int = 0, bias=None, out=None,
                    act_out=None, path: int = PATH_AUTO):
    """Quantise fp16 x [M, K] and apply the nested linear layer in one call.

    Returns (y fp32 [M, N], (xq, xscale, xsum)); the activation outputs are
    the same as quantize_act's.  `act_out` may supply their buffers."""
    import torch

    M, K = x.shape
    N = hi.shape[0]
    y = out if out is not None else torch.empty((M, N), dtype=torch.float32, device=x.device)
    if act_out is None:
        act_out = (torch.empty((M, K), dtype=torch.int8, device=x.device),
                   torch.empty((M,) if act_group == 0 else (M, K // GROUP), dtype=torch.float32,
                               device=x.device),
                   torch.empty((M, K // GROUP), dtype=torch.int32, device=x.device))
    xq, xs, xsum = act_out
    _check(lib().bitnest_quantize_linear(int(mode), _ptr(hi), _ptr(lo), _ptr(scale), _ptr(x), M, N,
                                         K, _ptr(y), int(act_group), _ptr(bias), _ptr(xq),
                                         _ptr(xs), _ptr(xsum), int(path), _stream(x)),
           "bitnest_quantize_linear")
    return y, (xq, xs, xsum)


def debug_group_sums(mode: int, hi, lo, xq, xsum, path: int = PATH_AUTO, out=None):
    """int32 [M, N, K/128] exact group sums, from the same inner loops as `linear`."""
    import torch

    M, K = xq.shape
    N = hi.shape[0]
    S = out if out is not None else torch.empty((M, N, K // GROUP), dtype=torch.int32,
                                                 device=xq.device)
    _check(lib().bitnest_debug_group_sums(int(mode), _ptr(hi), _ptr(lo), _ptr(xq), _ptr(xsum),
                                          M, N, K, _ptr(S), int(path), _stream(xq)),
           "bitnest_debug_group_sums")
    return S


# ------------------------------------------------- speculative decoding
class _SpecModelC(ctypes.Structure):
    _fields_ = [("vocab", ctypes.c_int64), ("dim", ctypes.c_int64), ("layers", ctypes.c_int64),
                ("embed", ctypes.c_void_p), ("hi", ctypes.POINTER(ctypes.c_void_p)),
                ("lo", ctypes.POINTER(ctypes.c_void_p)),
                ("scale", ctypes.POINTER(ctypes.c_void_p)), ("head_hi", ctypes.c_void_p),
                ("head_lo", ctypes.c_void_p), ("head_scale", ctypes.c_void_p)]


class SpecModel:
    """The synthetic model of bitnest_spec_rounds: embed fp16 [V, d] and
    (hi, lo, scale) device tensors per layer ([d, d/2] planes, [d, d/128]
    scales) and for the head ([V, d/2], [V, d/128]).  Holds the C struct."""

    def __init__(self, embed, layers, head):
        self.embed, self.layers, self.head = embed, list(layers), head
        self.vocab, self.dim = embed.shape
        n = len(self.layers)
        self._hi = (ctypes.c_void_p * max(n, 1))(*[t[0].data_ptr() for t in self.layers])
        self._lo = (ctypes.c_void_p * max(n, 1))(*[t[1].data_ptr() for t in self.layers])
        self._sc = (ctypes.c_void_p * max(n, 1))(*[t[2].data_ptr() for t in self.layers])
        self.c = _SpecModelC(self.vocab, self.dim, n, embed.data_ptr(),
                             ctypes.cast(self._hi, ctypes.POINTER(ctypes.c_void_p)),
                             ctypes.cast(self._lo, ctypes.POINTER(ctypes.c_void_p)),
                             ctypes.cast(self._sc, ctypes.POINTER(ctypes.c_void_p)),
                             head[0].data_ptr(), head[1].data_ptr(), head[2].data_ptr())


def spec_work_bytes(vocab: int, dim: int, gamma: int) -> int:
    n = lib().bitnest_spec_work_bytes(int(vocab), int(dim), int(gamma))
    if n < 0:
        _check(-n, "bitnest_spec_work_bytes")
    return n


def spec_rounds(model: SpecModel, gamma: int, rounds: int, seq, length, stats, work):
    """`rounds` speculative rounds on the device sequence `seq` (int32 [cap]),
    `length` (int32 [1]) and `stats` (int32 [4]), scratch `work` (uint8)."""
    _check(lib().bitnest_spec_rounds(ctypes.byref(model.c), int(gamma), int(rounds), _ptr(seq),
                                     seq.numel(), _ptr(length), _ptr(stats), _ptr(work),
                                     work.numel(), _stream(seq)), "bitnest_spec_rounds")


def spec_greedy(model: SpecModel, steps: int, seq, length, stats, work):
    """`steps` tokens of the target's greedy decoding, same buffers."""
    _check(lib().bitnest_spec_greedy(ctypes.byref(model.c), int(steps), _ptr(seq), seq.numel(),
                                     _ptr(length), _ptr(stats), _ptr(work), work.numel(),
                                     _stream(seq)), "bitnest_spec_greedy")
