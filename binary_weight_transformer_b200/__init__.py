"""B200-native low-bit-weight linear layer (BitNet-style BitLinear).

The operator and its sources are stated in ``include/lowbit.h``; every step
runs in the CUDA kernels of ``liblowbit.so`` (sm_100a).  This module only
marshals arguments: it takes torch tensors (device memory and the current
stream come from PyTorch), calls the C ABI through ctypes, and turns a
non-OK status into ``LowbitError``.  There is no CPU fallback: if the built
library is missing, importing a function raises.

Functions carry the ABI's names::

    packed, s_w = lowbit_pack(w, fmt, eps=1e-5)
    codes       = lowbit_unpack(packed, K, fmt)
    q, s_x      = lowbit_act_quant(x, eps=0.0)
    q, s_x      = lowbit_act_quant_ex(x, g=None, norm=NORM_RMS, eps_norm=1e-5, hadamard=0)
    y           = lowbit_linear(q, s_x, packed, s_w, fmt, N, out_dtype)
    y           = lowbit_bitlinear(x, packed, s_w, fmt, N, out_dtype, g=None, norm=NORM_RMS)
    ys          = lowbit_bitlinear_group(xs, packeds, s_ws, fmt, Ns, out_dtype)
"""
from __future__ import annotations

import ctypes
import os

TERNARY2, BINARY1, INT4 = 0, 1, 2
NORM_NONE, NORM_RMS = 0, 1
QUANT_DEFAULT, QUANT_BINARY_CENTRED = 0, 1
FUSED_MAX_BYTES = 98304  # LOWBIT_FUSED_MAX_BYTES
FUSED_MAX_K = 1024  # LOWBIT_FUSED_MAX_K
GROUP_MAX = 32  # LOWBIT_GROUP_MAX
F32, BF16, I32 = 0, 1, 2
WEIGHTS_STABLE = 1  # LOWBIT_LINEAR_WEIGHTS_STABLE
EXCLUSIVE = 2  # LOWBIT_LINEAR_EXCLUSIVE

STATUS_NAMES = {
    0: "LOWBIT_OK", 1: "LOWBIT_ERR_INVALID_ARG", 2: "LOWBIT_ERR_ALIGNMENT", 3: "LOWBIT_ERR_UNSUPPORTED",
    4: "LOWBIT_ERR_OVERFLOW_BOUND", 5: "LOWBIT_ERR_NONFINITE", 6: "LOWBIT_ERR_RESERVED_CODE",
    7: "LOWBIT_ERR_TIMEOUT", 8: "LOWBIT_ERR_CUDA",
}
OK, ERR_INVALID_ARG, ERR_ALIGNMENT, ERR_UNSUPPORTED, ERR_OVERFLOW_BOUND = 0, 1, 2, 3, 4
ERR_NONFINITE, ERR_RESERVED_CODE, ERR_TIMEOUT, ERR_CUDA = 5, 6, 7, 8

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblowbit.so")

# (name, restype, argtypes) of every entry point declared in include/lowbit.h
_P, _I64, _I32, _F, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
ABI = {
    "lowbit_packed_row_bytes": (_SZ, [_I32, _I64]),
    "lowbit_packed_ld": (_SZ, [_I32, _I64]),
    "lowbit_scale_count": (_I64, [_I32, _I64]),
    "lowbit_max_k": (_I64, [_I32]),
    "lowbit_pack_workspace_bytes": (_SZ, [_I32, _I64]),
    "lowbit_pack": (_I32, [_P, _I64, _I64, _I64, _I32, _F, _P, _I64, _P, _P, _SZ, _P, _P]),
    "lowbit_pack_ternary_noalloc": (_I32, [_P, _I64, _I64, _I64, _F, _P, _I64, _P, _P, _P]),
    "lowbit_unpack": (_I32, [_P, _I64, _I64, _I64, _I32, _P, _I64, _P, _P]),
    "lowbit_act_quant": (_I32, [_P, _I32, _I64, _I64, _I64, _F, _P, _I64, _P, _P, _P]),
    "lowbit_linear": (_I32, [_P, _I64, _P, _I64, _I64, _P, _I64, _P, _I32, _I64, _P, _I32, _I64, _P, _P]),
    "lowbit_linear_path": (_I32, [_P, _I64, _P, _I64, _I64, _P, _I64, _P, _I32, _I64, _P, _I32, _I64, _I32,
                                  _P, _P]),
    "lowbit_linear_ex": (_I32, [_P, _I64, _P, _I64, _I64, _P, _I64, _P, _I32, _I64, _P, _I32, _I64, _I32,
                                ctypes.c_uint, _P, _P]),
    "lowbit_linear_kernel": (_I32, [_I64, _I64, _I64, _I32, _I32, _I32, _P]),
    "lowbit_pack_ex_workspace_bytes": (_SZ, [_I32, _I32, _I64]),
    "lowbit_pack_ex": (_I32, [_P, _I64, _I64, _I64, _I32, _I32, _F, _P, _I64, _P, _P, _SZ, _P, _P]),
    "lowbit_act_row_stats": (_I32, [_P, _I32, _I64, _I64, _I64, _P, _I32, _P, _P, _P, _P]),
    "lowbit_act_quant_given_max": (_I32, [_P, _I32, _I64, _I64, _I64, _P, _I32, _P, _P, _I64, _P, _P]),
    "lowbit_act_scales": (_I32, [_P, _P, _I64, _I64, _I32, _F, _I32, _P, _P, _P]),
    "lowbit_rescale": (_I32, [_P, _I64, _I64, _I64, _P, _P, _I32, _P, _I32, _I64, _P, _P]),
    "lowbit_act_quant_ex": (_I32, [_P, _I32, _I64, _I64, _I64, _P, _I32, _F, _I32, _P, _I64, _P, _P, _P]),
    "lowbit_bitlinear": (_I32, [_P, _I32, _I64, _I64, _I64, _P, _I32, _F, _I32, _P, _I64, _P, _I32, _I64, _P, _I32,
                                _I64, _P, _I64, _P, _I32, ctypes.c_uint, _P, _P]),
    "lowbit_bitlinear_group": (_I32, [_P, _I32, _I64, _I32, _I32, _F, _I32, _I32, ctypes.c_uint, _P, _P]),
    "lowbit_kernel_name": (ctypes.c_char_p, [_I32]),
    "lowbit_status_string": (ctypes.c_char_p, [_I32]),
    "lowbit_set_wait_limit": (_I32, [_I64]),
    "lowbit_version": (_I32, []),
}


class LowbitError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m binary_weight_transformer_b200._build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in ABI.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _check(st: int, what: str):
    if st != OK:
        raise LowbitError(st, what)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def packed_row_bytes(fmt: int, K: int) -> int:
    return int(lib().lowbit_packed_row_bytes(fmt, K))


def packed_ld(fmt: int, K: int) -> int:
    return int(lib().lowbit_packed_ld(fmt, K))


def scale_count(fmt: int, N: int) -> int:
    return int(lib().lowbit_scale_count(fmt, N))


def max_k(fmt: int) -> int:
    return int(lib().lowbit_max_k(fmt))


def linear_kernel(M: int, N: int, K: int, fmt: int, path: int = 0, sm_count: int = 0) -> str:
    """Name of the kernel lowbit_linear (path 0) or a forced path launches for
    this problem on a GPU with `sm_count` SMs (0: the current device)."""
    k = ctypes.c_int(0)
    _check(lib().lowbit_linear_kernel(M, N, K, fmt, path, sm_count, ctypes.byref(k)), "lowbit_linear_kernel")
    return lib().lowbit_kernel_name(k.value).decode()


def status_flags(status_tensor) -> list[int]:
    """Decode a device status word (bit 1<<s per status s) into status values."""
    v = int(status_tensor.item())
    return [s for s in range(1, 9) if v & (1 << s)]


def lowbit_pack(w, fmt: int, eps: float = 1e-5, packed=None, s_w=None, ldp: int | None = None,
                workspace=None, status=None, stream=None):
    """Quantise and pack fp32 weights w[N, K] (CUDA tensor, unit inner stride)."""
    import torch
    N, K = w.shape
    if ldp is None:
        ldp = packed_ld(fmt, K)
    if packed is None:
        packed = torch.empty((N, ldp), dtype=torch.uint8, device=w.device)
    if s_w is None:
        s_w = torch.empty(scale_count(fmt, N), dtype=torch.float32, device=w.device)
    need = int(lib().lowbit_pack_workspace_bytes(fmt, N))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=w.device)
    st = lib().lowbit_pack(_ptr(w), N, K, w.stride(0), fmt, eps, _ptr(packed), packed.stride(0), _ptr(s_w),
                           _ptr(workspace), need, _ptr(status), _stream(stream))
    _check(st, "lowbit_pack")
    return packed, s_w


def lowbit_pack_ex(w, fmt: int, quantizer: int = QUANT_DEFAULT, eps: float = 1e-5, packed=None, s_w=None,
                   ldp: int | None = None, status=None, stream=None):
    """lowbit_pack with a choice of quantiser (QUANT_BINARY_CENTRED: BitNet v1
    centred sign codes, one scale mean|W| written to every row's entry)."""
    import torch
    N, K = w.shape
    if ldp is None:
        ldp = packed_ld(fmt, K)
    if packed is None:
        packed = torch.empty((N, ldp), dtype=torch.uint8, device=w.device)
    if s_w is None:
        s_w = torch.empty(scale_count(fmt, N), dtype=torch.float32, device=w.device)
    need = int(lib().lowbit_pack_ex_workspace_bytes(fmt, quantizer, N))
    workspace = torch.empty(need, dtype=torch.uint8, device=w.device) if need else None
    st = lib().lowbit_pack_ex(_ptr(w), N, K, w.stride(0), fmt, quantizer, eps, _ptr(packed), packed.stride(0),
                              _ptr(s_w), _ptr(workspace), need, _ptr(status), _stream(stream))
    _check(st, "lowbit_pack_ex")
    return packed, s_w


def lowbit_pack_ternary_noalloc(w, eps: float = 1e-5, packed=None, s_w=None, ldp: int | None = None,
                                status=None, stream=None):
    """Ternary pack that allocates nothing in the library (see lowbit.h);
    output tensors are still the caller's."""
    import torch
    N, K = w.shape
    if ldp is None:
        ldp = packed_ld(TERNARY2, K)
    if packed is None:
        packed = torch.empty((N, ldp), dtype=torch.uint8, device=w.device)
    if s_w is None:
        s_w = torch.empty(1, dtype=torch.float32, device=w.device)
    st = lib().lowbit_pack_ternary_noalloc(_ptr(w), N, K, w.stride(0), eps, _ptr(packed), packed.stride(0),
                                           _ptr(s_w), _ptr(status), _stream(stream))
    _check(st, "lowbit_pack_ternary_noalloc")
    return packed, s_w


def lowbit_unpack(packed, K: int, fmt: int, codes=None, status=None, stream=None):
    import torch
    N = packed.shape[0]
    if codes is None:
        codes = torch.empty((N, K), dtype=torch.int8, device=packed.device)
    st = lib().lowbit_unpack(_ptr(packed), packed.stride(0), N, K, fmt, _ptr(codes), codes.stride(0),
                             _ptr(status), _stream(stream))
    _check(st, "lowbit_unpack")
    return codes


def lowbit_act_quant(x, eps: float = 0.0, q=None, s_x=None, status=None, stream=None):
    """Per-token absmax int8 codes of x[M, K] (fp32 or bf16 CUDA tensor)."""
    import torch
    M, K = x.shape
    xdt = {torch.float32: F32, torch.bfloat16: BF16}[x.dtype]
    if q is None:
        q = torch.empty((M, (K + 15) // 16 * 16), dtype=torch.int8, device=x.device)
    if s_x is None:
        s_x = torch.empty(M, dtype=torch.float32, device=x.device)
    st = lib().lowbit_act_quant(_ptr(x), xdt, M, K, x.stride(0), eps, _ptr(q), q.stride(0), _ptr(s_x),
                                _ptr(status), _stream(stream))
    _check(st, "lowbit_act_quant")
    return q, s_x


def lowbit_linear(q, s_x, packed, s_w, fmt: int, N: int, out_dtype: int = F32, K: int | None = None,
                  y=None, status=None, stream=None, path: int = 0, weights_stable: bool = False,
                  exclusive: bool = False):
    """y[M, N] from int8 codes q[M, >=K] and a packed artifact (see lowbit.h).

    ``path`` 0 picks the kernel by M; 1 forces the GEMV, 2 the tensor-core GEMM
    with the expanded tile in shared memory, 3 the one with it in tensor memory,
    4 the tensor-memory one on SM pairs (256 weight rows per MMA), 5 the warp-level
    mma.sync kernel for at most 16 tokens, 6 the shared-memory one on SM pairs
    (256 tokens x 256 features per MMA).
    ``weights_stable`` passes LOWBIT_LINEAR_WEIGHTS_STABLE: the kernel that
    precedes this call on the stream does not write ``packed`` or ``s_w``, so
    weight reads may start before it finishes."""
    import torch
    M = q.shape[0]
    if K is None:
        K = q.shape[1]
    if y is None:
        dt = {F32: torch.float32, BF16: torch.bfloat16, I32: torch.int32}[out_dtype]
        y = torch.empty((M, N), dtype=dt, device=q.device)
    st = lib().lowbit_linear_ex(_ptr(q), q.stride(0), _ptr(s_x), M, K, _ptr(packed), packed.stride(0),
                                _ptr(s_w), fmt, N, _ptr(y), out_dtype, y.stride(0), path,
                                (WEIGHTS_STABLE if weights_stable else 0) | (EXCLUSIVE if exclusive else 0), _ptr(status), _stream(stream))
    _check(st, "lowbit_linear")
    return y


def _xdt(x):
    import torch
    return {torch.float32: F32, torch.bfloat16: BF16}[x.dtype]


def lowbit_act_quant_ex(x, g=None, norm: int = NORM_NONE, eps_norm: float = 1e-5, hadamard: int = 0, q=None,
                        s_x=None, status=None, stream=None):
    """Activation prologue of a BitLinear layer (see lowbit.h): gain g,
    RMSNorm, block Hadamard rotation, then per-token int8 codes."""
    import torch
    M, K = x.shape
    if q is None:
        q = torch.empty((M, (K + 15) // 16 * 16), dtype=torch.int8, device=x.device)
    if s_x is None:
        s_x = torch.empty(M, dtype=torch.float32, device=x.device)
    st = lib().lowbit_act_quant_ex(_ptr(x), _xdt(x), M, K, x.stride(0), _ptr(g), norm, eps_norm, hadamard,
                                   _ptr(q), q.stride(0), _ptr(s_x), _ptr(status), _stream(stream))
    _check(st, "lowbit_act_quant_ex")
    return q, s_x


def decodes_from_x(M: int, K: int, hadamard: int = 0, path: int = 0) -> bool:
    """True when the decode GEMV can take these token rows (lowbit_bitlinear_group)."""
    return M <= 4 and hadamard == 0 and path in (0, 1) and M * ((K + 127) // 128 * 128) <= FUSED_MAX_BYTES


def bitlinear_fuses(M: int, K: int, hadamard: int = 0, path: int = 0) -> bool:
    """True when lowbit_bitlinear runs as one fused decode kernel."""
    return decodes_from_x(M, K, hadamard, path) and K <= FUSED_MAX_K


def lowbit_bitlinear(x, packed, s_w, fmt: int, N: int, out_dtype: int = F32, g=None, norm: int = NORM_NONE,
                     eps_norm: float = 1e-5, hadamard: int = 0, y=None, q=None, s_x=None, want_codes: bool = False,
                     status=None, stream=None, path: int = 0, weights_stable: bool = False,
                     exclusive: bool = False):
    """The whole BitLinear forward from activations x[M, K] (fp32 or bf16).

    q and s_x are allocated as workspace when the call is not fused (or when
    ``want_codes``); returns y, or (y, q, s_x) with ``want_codes``."""
    import torch
    M, K = x.shape
    if y is None:
        dt = {F32: torch.float32, BF16: torch.bfloat16, I32: torch.int32}[out_dtype]
        y = torch.empty((M, N), dtype=dt, device=x.device)
    need = want_codes or not bitlinear_fuses(M, K, hadamard, path)
    if q is None and need:
        q = torch.empty((M, (K + 15) // 16 * 16), dtype=torch.int8, device=x.device)
    if s_x is None and need:
        s_x = torch.empty(M, dtype=torch.float32, device=x.device)
    st = lib().lowbit_bitlinear(_ptr(x), _xdt(x), M, K, x.stride(0), _ptr(g), norm, eps_norm, hadamard,
                                _ptr(packed), packed.stride(0), _ptr(s_w), fmt, N, _ptr(y), out_dtype, y.stride(0),
                                _ptr(q), q.stride(0) if q is not None else 0, _ptr(s_x), path,
                                (WEIGHTS_STABLE if weights_stable else 0) | (EXCLUSIVE if exclusive else 0), _ptr(status), _stream(stream))
    _check(st, "lowbit_bitlinear")
    return (y, q, s_x) if want_codes else y


class BitlinearItem(ctypes.Structure):
    """lowbit_bitlinear_item: one layer of a grouped decode call."""
    _fields_ = [("x", _P), ("ldx", _I64), ("g", _P), ("packed", _P), ("ldp", _I64), ("s_w", _P), ("N", _I64),
                ("K", _I64), ("y", _P), ("ldy", _I64), ("q", _P), ("ldq", _I64), ("s_x", _P)]


def lowbit_bitlinear_group(xs, packeds, s_ws, fmt: int, Ns, out_dtype: int = F32, gs=None, norm: int = NORM_NONE,
                           eps_norm: float = 1e-5, ys=None, want_codes: bool = False, status=None, stream=None,
                           weights_stable: bool = False, qs=None, s_xs=None, exclusive: bool = False):
    """Several independent decode BitLinear layers (M <= 4 tokens each, the
    same M, activation dtype, format and output dtype): the layers of at
    most FUSED_MAX_K features in one persistent fused GEMV launch, each
    longer layer as lowbit_bitlinear runs it (see lowbit.h).

    xs[i] [M, K_i], packeds[i], s_ws[i], Ns[i]; gs: None or a list of gains
    (entries may be None); qs / s_xs: optional per-layer code and scale
    buffers (allocated when the call needs them and they are not given).
    Returns the list of y, or (ys, qs, s_xs) with ``want_codes``."""
    import torch
    n = len(xs)
    if not (len(packeds) == len(s_ws) == len(Ns) == n) or (gs is not None and len(gs) != n):
        raise ValueError("every per-layer list must have one entry per layer")
    M = xs[0].shape[0]
    dt = {F32: torch.float32, BF16: torch.bfloat16, I32: torch.int32}[out_dtype]
    if ys is None:
        ys = [torch.empty((M, N), dtype=dt, device=x.device) for x, N in zip(xs, Ns)]
    # layers longer than FUSED_MAX_K run the prologue kernel, which writes
    # their codes: workspace then (allocated here unless given)
    if qs is None or s_xs is None:
        qs, s_xs = [None] * n, [None] * n
    if (want_codes or any(x.shape[1] > FUSED_MAX_K for x in xs)) and any(q is None for q in qs):
        qs = [torch.empty((M, (x.shape[1] + 15) // 16 * 16), dtype=torch.int8, device=x.device) for x in xs]
        s_xs = [torch.empty(M, dtype=torch.float32, device=x.device) for x in xs]
    items = (BitlinearItem * n)()
    for i in range(n):
        x, p, q, y = xs[i], packeds[i], qs[i], ys[i]
        if x.shape[0] != M or x.dtype != xs[0].dtype:
            raise ValueError("all layers take the same number of tokens and activation dtype")
        items[i] = BitlinearItem(_ptr(x), x.stride(0), _ptr(gs[i] if gs is not None else None), _ptr(p), p.stride(0),
                                 _ptr(s_ws[i]), Ns[i], x.shape[1], _ptr(y), y.stride(0), _ptr(q),
                                 q.stride(0) if q is not None else 0, _ptr(s_xs[i]))
    st = lib().lowbit_bitlinear_group(ctypes.cast(items, ctypes.c_void_p), n, M, _xdt(xs[0]), norm, eps_norm, fmt,
                                      out_dtype, (WEIGHTS_STABLE if weights_stable else 0) | (EXCLUSIVE if exclusive else 0), _ptr(status),
                                      _stream(stream))
    _check(st, "lowbit_bitlinear_group")
    return (ys, qs, s_xs) if want_codes else ys


def lowbit_act_row_stats(x, g=None, hadamard: int = 0, with_ss: bool = False, status=None, stream=None):
    """Per-row max|x*g| (fp32 [M]) and, with ``with_ss``, the fp64 sum of
    squares of a row slice (see lowbit.h, row-parallel layers)."""
    import torch
    M, K = x.shape
    row_max = torch.empty(M, dtype=torch.float32, device=x.device)
    row_ss = torch.empty(M, dtype=torch.float64, device=x.device) if with_ss else None
    st = lib().lowbit_act_row_stats(_ptr(x), _xdt(x), M, K, x.stride(0), _ptr(g), hadamard, _ptr(row_max),
                                    _ptr(row_ss), _ptr(status), _stream(stream))
    _check(st, "lowbit_act_row_stats")
    return row_max, row_ss


def lowbit_act_quant_given_max(x, row_max, g=None, hadamard: int = 0, q=None, status=None, stream=None):
    import torch
    M, K = x.shape
    if q is None:
        q = torch.empty((M, (K + 15) // 16 * 16), dtype=torch.int8, device=x.device)
    st = lib().lowbit_act_quant_given_max(_ptr(x), _xdt(x), M, K, x.stride(0), _ptr(g), hadamard, _ptr(row_max),
                                          _ptr(q), q.stride(0), _ptr(status), _stream(stream))
    _check(st, "lowbit_act_quant_given_max")
    return q


def lowbit_act_scales(row_max, row_ss, K_total: int, norm: int = NORM_NONE, eps_norm: float = 1e-5,
                      hadamard: int = 0, s_x=None, status=None, stream=None):
    import torch
    M = row_max.shape[0]
    if s_x is None:
        s_x = torch.empty(M, dtype=torch.float32, device=row_max.device)
    st = lib().lowbit_act_scales(_ptr(row_max), _ptr(row_ss), M, K_total, norm, eps_norm, hadamard, _ptr(s_x),
                                 _ptr(status), _stream(stream))
    _check(st, "lowbit_act_scales")
    return s_x


def lowbit_rescale(acc, s_x, s_w, fmt: int, out_dtype: int = F32, y=None, status=None, stream=None):
    """y = float(acc) * (s_w * s_x) from int32 accumulators acc[M, N]."""
    import torch
    M, N = acc.shape
    if y is None:
        dt = {F32: torch.float32, BF16: torch.bfloat16, I32: torch.int32}[out_dtype]
        y = torch.empty((M, N), dtype=dt, device=acc.device)
    st = lib().lowbit_rescale(_ptr(acc), acc.stride(0), M, N, _ptr(s_x), _ptr(s_w), fmt, _ptr(y), out_dtype,
                              y.stride(0), _ptr(status), _stream(stream))
    _check(st, "lowbit_rescale")
    return y


def set_wait_limit(cycles: int = 0):
    """Bound of the tensor-core kernels' pipeline waits on the current device
    (SM cycles; 0 restores the default).  See lowbit_set_wait_limit."""
    _check(lib().lowbit_set_wait_limit(cycles), "lowbit_set_wait_limit")
