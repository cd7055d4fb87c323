"""opt2s oracle: TEST INFRASTRUCTURE ONLY.

A ctypes front end to ``opt2s_oracle.c``, the plain single-threaded CPU
restatement of the 32-bit two-state optimizer update (Adam/AdamW, AdEMAMix).
Only the tests, the entry module's ``smoke()`` and the benchmark's CPU
baseline / reference legs may import this package; the library under
``elementwise_optimizer_b200`` never does, and the two share no code.

What it computes and where each step comes from is stated in the header of
``opt2s_oracle.c`` (bitsandbytes issue "Investigate a 256-thread SM103 path
for small 32-bit optimizer tensors", sections "Problem", "Scope" and
"Correctness oracle"; Kingma & Ba 2015 Algorithm 1; Loshchilov & Hutter 2019
Algorithm 2; Pagliardini et al. 2024 Algorithm 1; You et al. 2020 Algorithm 2
for LAMB).

Every function here was pinned by ``tests/test_oracle_pins.py`` against
values fixed by something other than the oracle itself (library optimizers in
float64, closed forms, invariants, numpy/ml_dtypes conversions).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "opt2s_oracle.c")
_LIB = os.path.join(_HERE, "libopt2s_oracle.so")

# Strict IEEE fp32: no contraction into FMA, no fast-math, SSE scalar float.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
          "-fno-fast-math", "-fexcess-precision=standard", "-mfpmath=sse",
          "-msse2"]

ALGO = {"adam": 0, "ademamix": 1}
DTYPE = {"f32": 0, "f16": 1, "bf16": 2}
_ITEMSIZE = {"f32": 4, "f16": 2, "bf16": 2}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (if missing or older than its source).

    ``OPT2S_ORACLE_LIB`` names a prebuilt library to load instead; the
    mutation test uses it to check that the pins reject broken oracles."""
    override = os.environ.get("OPT2S_ORACLE_LIB")
    if override:
        return override
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + ".tmp"
    subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    i64, i32, f32, f64, vp = (ctypes.c_int64, ctypes.c_int, ctypes.c_float,
                              ctypes.c_double, ctypes.c_void_p)
    lib.oracle_step_f32.argtypes = [i32, i32, i32, f32, f32, f32, f32, f32,
                                    f32, f32, i32, vp, vp, vp, vp, i64]
    lib.oracle_step_f32.restype = i32
    lib.oracle_step_f64.argtypes = [i32, i32, f64, f64, f64, f64, f64, f64,
                                    f64, i32, vp, vp, vp, vp, vp, i64]
    lib.oracle_step_f64.restype = i32
    lib.oracle_step_f32_fgrad.argtypes = [i32, i32, i32, f32, f32, f32, f32, f32,
                                          f32, f32, i32, vp, vp, vp, vp, i64]
    lib.oracle_step_f32_fgrad.restype = i32
    lib.oracle_step_f32_max_unorm.argtypes = [i32, i32, i32, f32, f32, f32, f32, f32,
                                              f32, f32, f32, i32, vp, vp, vp, vp, i64, vp]
    lib.oracle_step_f32_max_unorm.restype = i32
    lib.oracle_step_f32_lamb.argtypes = [i32, i32, f32, f32, f32, f32, f32, i32,
                                         vp, vp, vp, vp, i64, vp]
    lib.oracle_step_f32_lamb.restype = i32
    lib.oracle_quant_map.argtypes = [i32, vp]
    lib.oracle_quant_map.restype = i32
    lib.oracle_quantize.argtypes = [vp, f32]
    lib.oracle_quantize.restype = i32
    lib.oracle_step_8bit.argtypes = [i32, i32, i32, f32, f32, f32, f32, f32, f32, f32, i32,
                                     vp, vp, vp, vp, vp, vp, i64]
    lib.oracle_step_8bit.restype = i32
    lib.oracle_average_grads.argtypes = [i32, i32, vp, vp, i64]
    lib.oracle_average_grads.restype = i32
    lib.oracle_bias_correction.argtypes = [f32, i32]
    lib.oracle_bias_correction.restype = f32
    lib.oracle_decay_factor.argtypes = [f32, f32]
    lib.oracle_decay_factor.restype = f32
    lib.oracle_narrow_array.argtypes = [i32, vp, vp, i64]
    lib.oracle_narrow_array.restype = i32
    lib.oracle_widen_array.argtypes = [i32, vp, vp, i64]
    lib.oracle_widen_array.restype = i32
    _lib = lib
    return lib


def _ptr(a: np.ndarray | None) -> int | None:
    if a is None:
        return None
    if not a.flags["C_CONTIGUOUS"]:
        raise ValueError("oracle arrays must be C-contiguous")
    return a.ctypes.data


def step_f32(param: np.ndarray, grad: np.ndarray, state1: np.ndarray,
             state2: np.ndarray, *, dtype: str, algo: str, step: int,
             lr: float, beta1: float, beta2: float, eps: float,
             beta3: float = 0.0, alpha: float = 0.0,
             weight_decay: float = 0.0, skip_zeros: bool = False) -> None:
    """One fp32 optimizer step over one tensor, in place.

    ``param``/``grad`` hold the storage bits of ``dtype`` ('f32', 'f16',
    'bf16'; any numpy dtype of the right item size); ``state1`` holds m
    (Adam) or [m1 | m2] (AdEMAMix) as float32; ``state2`` holds v.
    """
    n = param.size
    if grad.size != n or param.itemsize != _ITEMSIZE[dtype] or \
            grad.itemsize != _ITEMSIZE[dtype]:
        raise ValueError("param/grad size or item size mismatch")
    want1 = 2 * n if algo == "ademamix" else n
    if state1.dtype != np.float32 or state2.dtype != np.float32 or \
            state1.size != want1 or state2.size != n:
        raise ValueError("state arrays must be float32 of the right length")
    rc = _load().oracle_step_f32(
        ALGO[algo], DTYPE[dtype], int(bool(skip_zeros)), lr, beta1, beta2,
        beta3, alpha, eps, weight_decay, int(step), _ptr(param), _ptr(grad),
        _ptr(state1), _ptr(state2), n)
    if rc != 0:
        raise ValueError(f"oracle_step_f32 rejected its arguments ({rc})")


def step_f32_max_unorm(param: np.ndarray, grad: np.ndarray, state1: np.ndarray,
                       state2: np.ndarray, *, dtype: str, algo: str, step: int,
                       lr: float, beta1: float, beta2: float, eps: float,
                       max_unorm: float, beta3: float = 0.0, alpha: float = 0.0,
                       weight_decay: float = 0.0, skip_zeros: bool = False) -> float:
    """One step over one tensor with its update norm clipped to
    max_unorm x its weight norm (max_unorm > 0); arrays as in step_f32.
    Returns the fp32 scale s the update was multiplied by (1 when the norm
    is within the bound)."""
    n = param.size
    if grad.size != n or param.itemsize != _ITEMSIZE[dtype] or \
            grad.itemsize != _ITEMSIZE[dtype]:
        raise ValueError("param/grad size or item size mismatch")
    want1 = 2 * n if algo == "ademamix" else n
    if state1.dtype != np.float32 or state2.dtype != np.float32 or \
            state1.size != want1 or state2.size != n:
        raise ValueError("state arrays must be float32 of the right length")
    scale = np.zeros(1, np.float32)
    rc = _load().oracle_step_f32_max_unorm(
        ALGO[algo], DTYPE[dtype], int(bool(skip_zeros)), lr, beta1, beta2,
        beta3, alpha, eps, weight_decay, max_unorm, int(step), _ptr(param), _ptr(grad),
        _ptr(state1), _ptr(state2), n, _ptr(scale))
    if rc != 0:
        raise ValueError(f"oracle_step_f32_max_unorm rejected its arguments ({rc})")
    return float(scale[0])


def step_f32_lamb(param: np.ndarray, grad: np.ndarray, m: np.ndarray,
                  v: np.ndarray, *, dtype: str, step: int, lr: float, beta1: float,
                  beta2: float, eps: float, weight_decay: float = 0.0,
                  skip_zeros: bool = False) -> float:
    """One LAMB step (You et al. 2020, Algorithm 2) over one tensor, in place:
    the Adam direction plus weight_decay * param, scaled by the trust ratio
    ||param|| / ||direction||.  ``param``/``grad`` hold storage bits of
    ``dtype``; ``m``, ``v`` are float32.  Returns the fp32 trust ratio."""
    n = param.size
    if grad.size != n or param.itemsize != _ITEMSIZE[dtype] or \
            grad.itemsize != _ITEMSIZE[dtype]:
        raise ValueError("param/grad size or item size mismatch")
    if m.dtype != np.float32 or v.dtype != np.float32 or m.size != n or v.size != n:
        raise ValueError("state arrays must be float32 of the param's size")
    ratio = np.zeros(1, np.float32)
    rc = _load().oracle_step_f32_lamb(
        DTYPE[dtype], int(bool(skip_zeros)), lr, beta1, beta2, eps, weight_decay,
        int(step), _ptr(param), _ptr(grad), _ptr(m), _ptr(v), n, _ptr(ratio))
    if rc != 0:
        raise ValueError(f"oracle_step_f32_lamb rejected its arguments ({rc})")
    return float(ratio[0])


BLOCK8 = 2048


def quant_map(signed: bool) -> np.ndarray:
    """The 256 values of the 8-bit state codes, ascending (signed: dynamic
    tree quantization for first moments; unsigned: for the second moment)."""
    out = np.empty(256, np.float32)
    if _load().oracle_quant_map(int(bool(signed)), _ptr(out)) != 0:
        raise ValueError("oracle_quant_map failed")
    return out


def quantize(qmap: np.ndarray, x) -> np.ndarray:
    """Codes of the map values nearest to x (ties to the lower code)."""
    qmap = np.ascontiguousarray(qmap, np.float32)
    xs = np.atleast_1d(np.asarray(x, np.float32))
    f = _load().oracle_quantize
    return np.array([f(_ptr(qmap), float(v)) for v in xs], np.uint8)


def step_8bit(param: np.ndarray, grad: np.ndarray, q1: np.ndarray, q2: np.ndarray,
              absmax1: np.ndarray, absmax2: np.ndarray, *, dtype: str, algo: str,
              step: int, lr: float, beta1: float, beta2: float, eps: float,
              beta3: float = 0.0, alpha: float = 0.0, weight_decay: float = 0.0,
              skip_zeros: bool = False) -> None:
    """One step over one tensor with 8-bit blockwise state, in place.
    q1: uint8 codes of m (n) or [m1 | m2] (2n); absmax1: float32 per block
    (nb) or [m1 | m2] (2 nb); q2: codes of v (n); absmax2: per block (nb)."""
    n = param.size
    nb = (n + BLOCK8 - 1) // BLOCK8
    two = algo == "ademamix"
    if grad.size != n or param.itemsize != _ITEMSIZE[dtype] or grad.itemsize != _ITEMSIZE[dtype]:
        raise ValueError("param/grad size or item size mismatch")
    if q1.dtype != np.uint8 or q2.dtype != np.uint8 or q1.size != (2 * n if two else n) or \
            q2.size != n:
        raise ValueError("codes must be uint8 of the right length")
    if absmax1.dtype != np.float32 or absmax2.dtype != np.float32 or \
            absmax1.size != (2 * nb if two else nb) or absmax2.size != nb:
        raise ValueError("absmax arrays must be float32 of the right length")
    rc = _load().oracle_step_8bit(
        ALGO[algo], DTYPE[dtype], int(bool(skip_zeros)), lr, beta1, beta2, beta3, alpha, eps,
        weight_decay, int(step), _ptr(param), _ptr(grad), _ptr(q1), _ptr(q2), _ptr(absmax1),
        _ptr(absmax2), n)
    if rc != 0:
        raise ValueError(f"oracle_step_8bit rejected its arguments ({rc})")


def step_f32_fgrad(param: np.ndarray, grad: np.ndarray, state1: np.ndarray,
                   state2: np.ndarray, *, dtype: str, algo: str, step: int,
                   lr: float, beta1: float, beta2: float, eps: float,
                   beta3: float = 0.0, alpha: float = 0.0,
                   weight_decay: float = 0.0, skip_zeros: bool = False) -> None:
    """``step_f32`` with a float32 gradient for a param of any storage dtype."""
    n = param.size
    if grad.dtype != np.float32 or grad.size != n or param.itemsize != _ITEMSIZE[dtype]:
        raise ValueError("grad must be float32 of the param's size")
    want1 = 2 * n if algo == "ademamix" else n
    if state1.dtype != np.float32 or state2.dtype != np.float32 or \
            state1.size != want1 or state2.size != n:
        raise ValueError("state arrays must be float32 of the right length")
    rc = _load().oracle_step_f32_fgrad(
        ALGO[algo], DTYPE[dtype], int(bool(skip_zeros)), lr, beta1, beta2,
        beta3, alpha, eps, weight_decay, int(step), _ptr(param), _ptr(grad),
        _ptr(state1), _ptr(state2), n)
    if rc != 0:
        raise ValueError(f"oracle_step_f32_fgrad rejected its arguments ({rc})")


def average_grads(grads: list, dtype: str) -> np.ndarray:
    """The rank-order fp32 mean of several ranks' gradients (storage bits of
    ``dtype``), as the sharded data-parallel step defines it."""
    n = grads[0].size
    arrs = [np.ascontiguousarray(g) for g in grads]
    for a in arrs:
        if a.size != n or a.itemsize != _ITEMSIZE[dtype]:
            raise ValueError("gradients must share size and storage dtype")
    ptrs = (ctypes.c_void_p * len(arrs))(*[a.ctypes.data for a in arrs])
    out = np.empty(n, np.float32)
    rc = _load().oracle_average_grads(DTYPE[dtype], len(arrs), ctypes.cast(ptrs, ctypes.c_void_p),
                                      _ptr(out), n)
    if rc != 0:
        raise ValueError("oracle_average_grads rejected its arguments")
    return out


def step_f64(param: np.ndarray, grad: np.ndarray, m: np.ndarray,
             v: np.ndarray, m2: np.ndarray | None = None, *, algo: str,
             step: int, lr: float, beta1: float, beta2: float, eps: float,
             beta3: float = 0.0, alpha: float = 0.0,
             weight_decay: float = 0.0, skip_zeros: bool = False) -> None:
    """The float64 shadow of ``step_f32`` (same definitions, all in double)."""
    arrs = [param, grad, m, v] + ([m2] if m2 is not None else [])
    for a in arrs:
        if a.dtype != np.float64 or a.size != param.size:
            raise ValueError("shadow arrays must be float64 of equal size")
    rc = _load().oracle_step_f64(
        ALGO[algo], int(bool(skip_zeros)), lr, beta1, beta2, beta3, alpha,
        eps, weight_decay, int(step), _ptr(param), _ptr(grad), _ptr(m),
        _ptr(m2), _ptr(v), param.size)
    if rc != 0:
        raise ValueError(f"oracle_step_f64 rejected its arguments ({rc})")


def bias_correction(beta: float, t: int) -> float:
    return _load().oracle_bias_correction(beta, t)


def decay_factor(lr: float, wd: float) -> float:
    return _load().oracle_decay_factor(lr, wd)


def narrow(x: np.ndarray, dtype: str) -> np.ndarray:
    """float32 -> fp16/bf16 bit patterns (uint16), round-to-nearest-even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    _load().oracle_narrow_array(DTYPE[dtype], _ptr(x), _ptr(out), x.size)
    return out


def widen(h: np.ndarray, dtype: str) -> np.ndarray:
    """fp16/bf16 bit patterns (uint16) -> float32, exact."""
    h = np.ascontiguousarray(h).view(np.uint16)
    out = np.empty(h.shape, np.float32)
    _load().oracle_widen_array(DTYPE[dtype], _ptr(h), _ptr(out), h.size)
    return out
