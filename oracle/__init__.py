"""The oracle: a plain CPU statement of the low-bit-weight linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this package.  The CUDA library never imports it, and it never imports the
CUDA library.

The arithmetic lives in ``lowbit_oracle.c`` (scalar C, ``-O2
-ffp-contract=off``); this module builds it with gcc into
``oracle/_build/liblowbit_oracle.so`` and wraps each function with numpy
arrays.  Every function raises ``OracleError`` with the C status on failure.

Sources (page title and section): "M8.8 - Native Binary and Ternary
Transformers" §0x02C-0x02E, §0x05A-0x05D, §0x06E, §0x09C; "Atomic-1Bit"
README opening section; "T4NT-0.5B" model card, Architecture table.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lowbit_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "liblowbit_oracle.so")

TERNARY2, BINARY1, INT4 = 0, 1, 2
OK, EINVAL, EOVERFLOW, ENONFINITE, ERESERVED = 0, 1, 4, 5, 6


class OracleError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"oracle {what} failed with status {status}")
        self.status = status


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP on) unless an up-to-date build exists."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        L = ctypes.c_long
        I = ctypes.c_int
        F = ctypes.c_float
        sig = {
            "orc_ternary_codes": [P, L, L, L, F, P, P],
            "orc_binary_codes": [P, L, L, L, P, P],
            "orc_int4_codes": [P, L, L, L, P, P],
            "orc_pack": [P, L, L, I, P, L],
            "orc_unpack": [P, L, L, L, I, P],
            "orc_act_quant_f32": [P, L, L, L, F, P, L, P],
            "orc_act_quant_bf16": [P, L, L, L, F, P, L, P],
            "orc_int_dot": [P, L, P, L, L, L, I, P, I],
            "orc_rescale_f32": [P, L, L, P, L, P, P, L],
            "orc_rescale_bf16": [P, L, L, P, L, P, P, L],
            "orc_max_threads": [],
            "orc_binary_centred_codes": [P, L, L, L, P, P, P],
            "orc_act_prologue_f32": [P, L, L, L, P, I, F, L, P, L, P],
            "orc_act_prologue_bf16": [P, L, L, L, P, I, F, L, P, L, P],
        }
        for name, args in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = I
        lib.orc_tanh.argtypes = [ctypes.c_double]
        lib.orc_tanh.restype = ctypes.c_double
        lib.orc_row_bytes.argtypes = [I, L]
        lib.orc_row_bytes.restype = L
        lib.orc_f32_to_bf16.argtypes = [F]
        lib.orc_f32_to_bf16.restype = ctypes.c_uint16
        lib.orc_fwht32.argtypes = [P, L]
        lib.orc_fwht32.restype = None
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(st: int, what: str):
    if st != OK:
        raise OracleError(st, what)


def max_threads() -> int:
    return _load().orc_max_threads()


def tanh(z: float) -> float:
    """The oracle's own fp64 tanh (see lowbit_oracle.c)."""
    return _load().orc_tanh(float(z))


def f32_to_bf16_bits(y: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest even) bit patterns, element by element."""
    lib = _load()
    flat = np.ascontiguousarray(y, dtype=np.float32).ravel()
    out = np.empty(flat.shape, np.uint16)
    for i, v in enumerate(flat):
        out[i] = lib.orc_f32_to_bf16(float(v))
    return out.reshape(np.shape(y))


def ternary_codes(w: np.ndarray, eps: float = 1e-5):
    """Absmean ternary codes and the per-tensor scale gamma (M8.8 §0x05A)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.empty((N, K), np.int8)
    gamma = np.zeros(1, np.float32)
    _check(_load().orc_ternary_codes(_p(w), N, K, K, ctypes.c_float(eps), _p(codes), _p(gamma)),
           "ternary_codes")
    return codes, gamma


def binary_codes(w: np.ndarray):
    """Sign codes (+1 for w >= 0) and per-row mean|W| scales (M8.8 §0x06E)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.empty((N, K), np.int8)
    s_w = np.empty(N, np.float32)
    _check(_load().orc_binary_codes(_p(w), N, K, K, _p(codes), _p(s_w)), "binary_codes")
    return codes, s_w


def int4_codes(w: np.ndarray):
    """3*tanh(w/3) clipping then per-row 15-level codes (T4NT-0.5B)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.empty((N, K), np.int8)
    s_w = np.empty(N, np.float32)
    _check(_load().orc_int4_codes(_p(w), N, K, K, _p(codes), _p(s_w)), "int4_codes")
    return codes, s_w


def binary_centred_codes(w: np.ndarray):
    """BitNet v1 centred sign codes (+1 where w > mean(W), else -1) and the
    per-tensor scale beta = mean|W| (M8.8 §0x02B, §0x02E).  Returns
    (codes, beta[1], alpha[1])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.empty((N, K), np.int8)
    alpha = np.zeros(1, np.float32)
    beta = np.zeros(1, np.float32)
    _check(_load().orc_binary_centred_codes(_p(w), N, K, K, _p(codes), _p(alpha), _p(beta)),
           "binary_centred_codes")
    return codes, beta, alpha


def fwht32(v: np.ndarray) -> np.ndarray:
    """Unnormalised fast Walsh-Hadamard transform of each row of v (fp32,
    row length a power of two), radix-2, stages h = 1, 2, ... (M8.8 §0x07C)."""
    v = np.array(v, dtype=np.float32, order="C", copy=True)
    n = v.shape[-1]
    assert n > 0 and n & (n - 1) == 0
    flat = v.reshape(-1, n)
    for r in range(flat.shape[0]):
        row = flat[r]
        _load().orc_fwht32(row.ctypes.data_as(ctypes.c_void_p), n)
    return v


def act_prologue(x: np.ndarray, g: np.ndarray | None = None, norm: bool = False, eps_norm: float = 1e-5,
                 hadamard: int = 0, bf16_bits: bool = False):
    """RMSNorm (norm=True) with gain g, optional block Hadamard rotation of
    block size `hadamard`, then per-token absmax int8 codes; returns (q, s_x).
    The codes come from FWHT(x*g) and the row factors 1/rms and
    1/sqrt(hadamard) enter the scale only (see lowbit_oracle.c)."""
    if bf16_bits:
        x = np.ascontiguousarray(x, dtype=np.uint16)
        fn = _load().orc_act_prologue_bf16
    else:
        x = np.ascontiguousarray(x, dtype=np.float32)
        fn = _load().orc_act_prologue_f32
    M, K = x.shape
    gp = None
    if g is not None:
        g = np.ascontiguousarray(g, dtype=np.float32)
        assert g.shape == (K,)
        gp = _p(g)
    q = np.empty((M, K), np.int8)
    s_x = np.empty(M, np.float32)
    _check(fn(_p(x), M, K, K, gp, 1 if norm else 0, ctypes.c_float(eps_norm), hadamard, _p(q), K, _p(s_x)),
           "act_prologue")
    return q, s_x


def quantize(w: np.ndarray, fmt: int, eps: float = 1e-5):
    if fmt == TERNARY2:
        return ternary_codes(w, eps)
    if fmt == BINARY1:
        return binary_codes(w)
    if fmt == INT4:
        return int4_codes(w)
    raise ValueError(fmt)


def row_bytes(fmt: int, K: int) -> int:
    return int(_load().orc_row_bytes(fmt, K))


def pack(codes: np.ndarray, fmt: int, ldp: int | None = None) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    N, K = codes.shape
    if ldp is None:
        ldp = row_bytes(fmt, K)
    out = np.empty((N, ldp), np.uint8)
    _check(_load().orc_pack(_p(codes), N, K, fmt, _p(out), ldp), "pack")
    return out


def unpack(packed: np.ndarray, K: int, fmt: int):
    """Returns (codes, status); status is ERESERVED if a reserved pattern or a
    non-zero padding bit was found."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N, ldp = packed.shape
    codes = np.empty((N, K), np.int8)
    st = _load().orc_unpack(_p(packed), ldp, N, K, fmt, _p(codes))
    if st not in (OK, ERESERVED):
        raise OracleError(st, "unpack")
    return codes, st


def act_quant(x: np.ndarray, eps: float = 0.0, bf16_bits: bool = False):
    """Per-token absmax int8 codes q and scales s_x (M8.8 §0x05C).

    ``x`` is fp32, or uint16 bf16 bit patterns when ``bf16_bits``."""
    if bf16_bits:
        x = np.ascontiguousarray(x, dtype=np.uint16)
        fn = _load().orc_act_quant_bf16
    else:
        x = np.ascontiguousarray(x, dtype=np.float32)
        fn = _load().orc_act_quant_f32
    M, K = x.shape
    q = np.empty((M, K), np.int8)
    s_x = np.empty(M, np.float32)
    _check(fn(_p(x), M, K, K, ctypes.c_float(eps), _p(q), K, _p(s_x)), "act_quant")
    return q, s_x


def int_dot(q: np.ndarray, codes: np.ndarray, fmt: int, nthreads: int = 1) -> np.ndarray:
    """acc[t,n] = sum_k q[t,k]*c[n,k] in int64 by the add/sub/skip rule."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    M, K = q.shape
    N = codes.shape[0]
    assert codes.shape[1] == K
    acc = np.empty((M, N), np.int64)
    _check(_load().orc_int_dot(_p(q), K, _p(codes), M, N, K, fmt, _p(acc), nthreads), "int_dot")
    return acc


def rescale(acc: np.ndarray, s_w: np.ndarray, s_x: np.ndarray, out: str = "f32") -> np.ndarray:
    """y = float(acc) * (s_w * s_x); ``out`` is "f32" or "bf16" (uint16 bits)."""
    acc = np.ascontiguousarray(acc, dtype=np.int64)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32).ravel()
    s_x = np.ascontiguousarray(s_x, dtype=np.float32).ravel()
    M, N = acc.shape
    if out == "f32":
        y = np.empty((M, N), np.float32)
        fn = _load().orc_rescale_f32
    elif out == "bf16":
        y = np.empty((M, N), np.uint16)
        fn = _load().orc_rescale_bf16
    else:
        raise ValueError(out)
    _check(fn(_p(acc), M, N, _p(s_w), s_w.size, _p(s_x), _p(y), N), "rescale")
    return y


def linear(q: np.ndarray, s_x: np.ndarray, packed: np.ndarray, s_w: np.ndarray, fmt: int,
           K: int, out: str = "f32", nthreads: int = 1):
    """Whole operator on a packed artifact: unpack -> int dot -> rescale.

    Returns (y, acc)."""
    codes, st = unpack(packed, K, fmt)
    if st != OK:
        raise OracleError(st, "linear/unpack")
    acc = int_dot(q, codes, fmt, nthreads)
    return rescale(acc, s_w, s_x, out), acc
