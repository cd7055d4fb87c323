"""Thin ctypes binding of libopt2s.so (include/opt2s.h).

Argument marshalling only: every step of the optimizer update runs in the CUDA
kernels of libopt2s.so.  There is no CPU fallback -- if the library is missing
or cannot be loaded, every call raises.  PyTorch is used by callers only for
device memory and streams; the binding takes raw device pointers or torch
tensors (for which it reads ``data_ptr()``, ``numel()`` and ``dtype``).
"""
from __future__ import annotations

import contextlib
import ctypes
import os
from typing import Iterable, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libopt2s.so")
# the test build: the same kernels plus the forcing knobs, the fault
# injection and the division check (tests only, through testing_library())
TESTING_LIB_PATH = os.path.join(_PKG, "libopt2s_testing.so")

OPT2S_F32, OPT2S_F16, OPT2S_BF16 = 0, 1, 2
OPT2S_ADAM, OPT2S_ADEMAMIX = 0, 1
ALGOS = {"adam": OPT2S_ADAM, "adamw": OPT2S_ADAM, "ademamix": OPT2S_ADEMAMIX}
DTYPES = {"f32": OPT2S_F32, "f16": OPT2S_F16, "bf16": OPT2S_BF16}

OPT2S_OK = 0
STATUS = {0: "OPT2S_OK", -1: "OPT2S_ERR_INVALID_ARG", -2: "OPT2S_ERR_ALIAS",
          -3: "OPT2S_ERR_NO_MEMORY", -4: "OPT2S_ERR_CUDA",
          -5: "OPT2S_ERR_DEVICE", -6: "OPT2S_ERR_TOO_LARGE"}


class Opt2sError(RuntimeError):
    def __init__(self, status: int, where: str, cuda_error: int = 0):
        self.status = status
        self.cuda_error = cuda_error
        msg = f"{where}: {STATUS.get(status, status)} ({_error_string(status)})"
        if status == -4:
            msg += f", cudaError {cuda_error}"
        super().__init__(msg)


class opt2s_tensor(ctypes.Structure):
    _fields_ = [("param", ctypes.c_void_p), ("grad", ctypes.c_void_p),
                ("state1", ctypes.c_void_p), ("state2", ctypes.c_void_p),
                ("numel", ctypes.c_int64), ("dtype", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class TensorListDesc(ctypes.Structure):
    _fields_ = [("tensors", ctypes.POINTER(opt2s_tensor)), ("count", ctypes.c_int32)]


class Hyper(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float),
                ("beta2", ctypes.c_float), ("beta3", ctypes.c_float),
                ("alpha", ctypes.c_float), ("eps", ctypes.c_float),
                ("weight_decay", ctypes.c_float), ("algo", ctypes.c_int32),
                ("skip_zeros", ctypes.c_int32)]


class opt2s_step_scalars(ctypes.Structure):
    _fields_ = [(n, ctypes.c_float) for n in (
        "lr", "beta1", "beta2", "beta3", "one_minus_beta1", "one_minus_beta2",
        "one_minus_beta3", "alpha", "eps", "bc1", "bc2", "decay")] + [
        ("inv_bc1", ctypes.c_double), ("inv_bc2", ctypes.c_double)] + [
        (n, ctypes.c_float) for n in ("rcp_bc1_hi", "rcp_bc1_lo", "rcp_bc2_hi", "rcp_bc2_lo")]


MAX_WORLD = 8


class opt2s_shard_desc(ctypes.Structure):
    _fields_ = [("world", ctypes.c_int32), ("rank", ctypes.c_int32), ("numel", ctypes.c_int64),
                ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("params", ctypes.c_void_p * MAX_WORLD), ("grads", ctypes.c_void_p * MAX_WORLD),
                ("state1", ctypes.c_void_p), ("state2", ctypes.c_void_p)]


class opt2s_tensor8(ctypes.Structure):
    _fields_ = [("param", ctypes.c_void_p), ("grad", ctypes.c_void_p),
                ("state1", ctypes.c_void_p), ("state2", ctypes.c_void_p),
                ("absmax1", ctypes.c_void_p), ("absmax2", ctypes.c_void_p),
                ("numel", ctypes.c_int64), ("dtype", ctypes.c_int32),
                ("state_bits", ctypes.c_int32)]


class TensorListDesc8(ctypes.Structure):
    _fields_ = [("tensors", ctypes.POINTER(opt2s_tensor8)), ("count", ctypes.c_int32)]


BLOCK8 = 2048
MIN_8BIT_SIZE = 4096


class opt2s_ipc_handle(ctypes.Structure):
    _fields_ = [("bytes", ctypes.c_ubyte * 64)]


class opt2s_testing_chunk(ctypes.Structure):
    _fields_ = [("tensor", ctypes.c_int64), ("start", ctypes.c_int64),
                ("len", ctypes.c_int64), ("dtype", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


EXPORTS = {
    # name: (restype, argtypes)
    "opt2s_step": (ctypes.c_int, [ctypes.POINTER(TensorListDesc), ctypes.POINTER(Hyper),
                                  ctypes.c_int, ctypes.c_void_p]),
    "opt2s_plan_create": (ctypes.c_int, [ctypes.POINTER(TensorListDesc), ctypes.c_int32,
                                         ctypes.POINTER(ctypes.c_void_p)]),
    "opt2s_plan_step": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(Hyper), ctypes.c_int,
                                       ctypes.c_void_p]),
    "opt2s_plan_destroy": (ctypes.c_int, [ctypes.c_void_p]),
    "opt2s_plan_num_chunks": (ctypes.c_int64, [ctypes.c_void_p]),
    "opt2s_step_noalloc": (ctypes.c_int, [ctypes.POINTER(TensorListDesc), ctypes.POINTER(Hyper),
                                          ctypes.c_int, ctypes.c_void_p]),
    "opt2s_noalloc_max_chunks": (ctypes.c_int64, []),
    "opt2s_step_max_unorm": (ctypes.c_int, [ctypes.POINTER(TensorListDesc), ctypes.POINTER(Hyper),
                                            ctypes.c_float, ctypes.c_int, ctypes.c_void_p]),
    "opt2s_step_lamb": (ctypes.c_int, [ctypes.POINTER(TensorListDesc), ctypes.POINTER(Hyper),
                                       ctypes.c_int, ctypes.c_void_p]),
    "opt2s_step_8bit": (ctypes.c_int, [ctypes.POINTER(TensorListDesc8), ctypes.POINTER(Hyper),
                                       ctypes.c_int, ctypes.c_void_p]),
    "opt2s_8bit_state_bits": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64]),
    "opt2s_fill_step_scalars": (ctypes.c_int, [ctypes.POINTER(Hyper), ctypes.c_int, ctypes.c_int,
                                               ctypes.c_void_p]),
    "opt2s_plan_step_table": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                             ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]),
    "opt2s_shard_range": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                         ctypes.POINTER(ctypes.c_int64),
                                         ctypes.POINTER(ctypes.c_int64)]),
    "opt2s_shard_step": (ctypes.c_int, [ctypes.POINTER(opt2s_shard_desc), ctypes.POINTER(Hyper),
                                        ctypes.c_int, ctypes.c_void_p]),
    "opt2s_ipc_export": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(opt2s_ipc_handle),
                                        ctypes.POINTER(ctypes.c_int64)]),
    "opt2s_ipc_open": (ctypes.c_int, [ctypes.POINTER(opt2s_ipc_handle), ctypes.c_int64,
                                      ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_void_p)]),
    "opt2s_ipc_close": (ctypes.c_int, [ctypes.c_void_p]),
    "opt2s_release_cache": (ctypes.c_int, []),
    "opt2s_error_string": (ctypes.c_char_p, [ctypes.c_int]),
    "opt2s_last_cuda_error": (ctypes.c_int, []),
    "opt2s_abi_version": (ctypes.c_int, []),
    "opt2s_testing_build_chunks": (ctypes.c_int, [ctypes.POINTER(TensorListDesc), ctypes.c_int32,
                                                  ctypes.c_int64,
                                                  ctypes.POINTER(opt2s_testing_chunk),
                                                  ctypes.c_int64, ctypes.POINTER(ctypes.c_int64)]),
    "opt2s_testing_validate": (ctypes.c_int, [ctypes.POINTER(TensorListDesc),
                                              ctypes.POINTER(Hyper), ctypes.c_int]),
    "opt2s_testing_unorm_tables": (ctypes.c_int, [ctypes.POINTER(TensorListDesc), ctypes.c_int32,
                                                  ctypes.c_int64, ctypes.POINTER(ctypes.c_uint32),
                                                  ctypes.POINTER(ctypes.c_uint32),
                                                  ctypes.POINTER(ctypes.c_uint32),
                                                  ctypes.POINTER(ctypes.c_int64)]),
    "opt2s_testing_set_chunk_elems": (ctypes.c_int64, [ctypes.c_int64]),
    "opt2s_testing_set_launch": (ctypes.c_int, [ctypes.c_int, ctypes.c_int]),
    "opt2s_testing_default_chunk_elems": (ctypes.c_int64, []),
    "opt2s_testing_launch_count": (ctypes.c_int64, []),
    "opt2s_testing_fail_allocs": (ctypes.c_int, [ctypes.c_int]),
    "opt2s_testing_choose_chunk_elems": (ctypes.c_int64, [ctypes.POINTER(TensorListDesc),
                                                          ctypes.c_int64]),
    "opt2s_testing_check_division": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32,
                                                    ctypes.POINTER(ctypes.c_int64)]),
    "opt2s_testing_max_block_threads": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32]),
    "opt2s_testing_quant_tables": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int64]),
}

# exported by the test build only
TESTING_ONLY = {"opt2s_testing_set_chunk_elems", "opt2s_testing_set_launch",
                "opt2s_testing_fail_allocs", "opt2s_testing_check_division"}

_libs = {}
_use_testing = False


def _load(path: str, testing: bool) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build the CUDA library first "
            "(python -m elementwise_optimizer_b200._build); there is no CPU fallback")
    L = ctypes.CDLL(path)
    for name, (res, args) in EXPORTS.items():
        if name in TESTING_ONLY and not testing:
            continue
        fn = getattr(L, name)
        fn.restype, fn.argtypes = res, args
    return L


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built): libopt2s.so, or
    the test build inside ``testing_library()``."""
    key = "testing" if _use_testing else "product"
    if key not in _libs:
        _libs[key] = _load(TESTING_LIB_PATH if _use_testing else LIB_PATH, _use_testing)
    return _libs[key]


@contextlib.contextmanager
def testing_library():
    """Route every call of this module to the test build of the library
    (libopt2s_testing.so: the same kernels, plus the forcing knobs and the
    fault injection).  Tests only; plans made inside stay bound to it.  On
    exit the knobs are reset and its plan cache released."""
    global _use_testing
    prev = _use_testing
    _use_testing = True
    try:
        yield lib()
    finally:
        try:
            L = lib()
            L.opt2s_testing_set_launch(0, 0)
            L.opt2s_testing_set_chunk_elems(0)
            L.opt2s_testing_fail_allocs(0)
            L.opt2s_release_cache()
        finally:
            _use_testing = prev


def _testing_lib() -> ctypes.CDLL:
    if not _use_testing:
        raise RuntimeError("forcing knobs and fault injection exist only in the test build: "
                           "call them inside binding.testing_library()")
    return lib()


def _error_string(status: int) -> str:
    try:
        return lib().opt2s_error_string(status).decode()
    except Exception:  # pragma: no cover - only while formatting an error
        return "?"


def check(status: int, where: str, L: ctypes.CDLL | None = None) -> None:
    """Raise Opt2sError for a failed call (L: the library that made it)."""
    if status != OPT2S_OK:
        raise Opt2sError(status, where, (L or lib()).opt2s_last_cuda_error())


# ---------------------------------------------------------------------------
# Marshalling
# ---------------------------------------------------------------------------

def _torch_dtype_code(t) -> int:
    import torch
    code = {torch.float32: OPT2S_F32, torch.float16: OPT2S_F16,
            torch.bfloat16: OPT2S_BF16}.get(t.dtype)
    if code is None:
        raise TypeError(f"unsupported param dtype {t.dtype}")
    return code


def _ptr(x) -> int:
    return x if isinstance(x, int) else int(x.data_ptr())


class TensorList:
    """A marshalled collection: the ctypes descriptor a step is called with.

    Build it once and reuse it: the records hold raw device pointers, so the
    tensors must stay alive (and in place) while the list is used.
    """

    def __init__(self, records: Sequence[tuple]):
        """records: (param, grad, state1, state2, numel, dtype_code) tuples,
        the pointers as ints."""
        n = len(records)
        self._arr = (opt2s_tensor * max(n, 1))()
        for i, (p, g, s1, s2, numel, dt) in enumerate(records):
            self._arr[i] = opt2s_tensor(p, g, s1, s2, int(numel), int(dt), 0)
        self.desc = TensorListDesc(ctypes.cast(self._arr, ctypes.POINTER(opt2s_tensor)), n)
        self.count = n

    @classmethod
    def from_tensors(cls, params: Iterable, grads: Iterable, state1: Iterable,
                     state2: Iterable) -> "TensorList":
        """From torch tensors (contiguous, on the same CUDA device)."""
        recs = []
        for p, g, s1, s2 in zip(params, grads, state1, state2):
            for t in (p, g, s1, s2):
                if not t.is_contiguous():
                    raise ValueError("tensors must be contiguous")
            if g.dtype != p.dtype or g.numel() != p.numel():
                raise ValueError("grad must match param in dtype and size")
            recs.append((_ptr(p), _ptr(g), _ptr(s1), _ptr(s2), p.numel(),
                         _torch_dtype_code(p)))
        return cls(recs)


class TensorList8:
    """A marshalled collection for the 8-bit-state step: records (param,
    grad, state1, state2, absmax1, absmax2, numel, dtype_code, state_bits),
    pointers as ints (absmax pointers 0 for 32-bit records)."""

    def __init__(self, records: Sequence[tuple]):
        n = len(records)
        self._arr = (opt2s_tensor8 * max(n, 1))()
        for i, (p, g, s1, s2, a1, a2, numel, dt, bits) in enumerate(records):
            self._arr[i] = opt2s_tensor8(p, g, s1, s2, a1 or None, a2 or None, int(numel),
                                         int(dt), int(bits))
        self.desc = TensorListDesc8(ctypes.cast(self._arr, ctypes.POINTER(opt2s_tensor8)), n)
        self.count = n

    @classmethod
    def from_tensors(cls, params, grads, state1, state2, absmax1, absmax2) -> "TensorList8":
        """From torch tensors; a record is 8-bit when its state1 is uint8
        (then absmax1/absmax2 are its fp32 block absmaxes), else 32-bit
        (absmax entries None)."""
        import torch
        recs = []
        for p, g, s1, s2, a1, a2 in zip(params, grads, state1, state2, absmax1, absmax2):
            for t in (p, g, s1, s2) + tuple(x for x in (a1, a2) if x is not None):
                if not t.is_contiguous():
                    raise ValueError("tensors must be contiguous")
            if g.dtype != p.dtype or g.numel() != p.numel():
                raise ValueError("grad must match param in dtype and size")
            eight = s1.dtype == torch.uint8
            if eight != (a1 is not None and a2 is not None):
                raise ValueError("8-bit records need both absmax tensors, 32-bit ones none")
            recs.append((_ptr(p), _ptr(g), _ptr(s1), _ptr(s2), _ptr(a1) if eight else 0,
                         _ptr(a2) if eight else 0, p.numel(), _torch_dtype_code(p),
                         8 if eight else 32))
        return cls(recs)


def make_hyper(algo: str = "adam", lr: float = 1e-3, beta1: float = 0.9,
               beta2: float = 0.999, eps: float = 1e-8, weight_decay: float = 0.0,
               beta3: float = 0.0, alpha: float = 0.0, skip_zeros: bool = False) -> Hyper:
    return Hyper(lr, beta1, beta2, beta3, alpha, eps, weight_decay, ALGOS[algo],
                 int(bool(skip_zeros)))


def _current_stream_fast():
    """Raw handle of torch's current stream on the current device.  Building
    a torch.cuda.Stream object costs microseconds per call, so the private
    raw-handle query is used when this torch build has it."""
    import torch
    get_raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
    get_dev = getattr(torch._C, "_cuda_getDevice", None)
    if get_raw is not None and get_dev is not None:
        return int(get_raw(get_dev()))
    return int(torch.cuda.current_stream().cuda_stream)


def _stream_handle(stream) -> int:
    if stream is None:
        return _current_stream_fast()
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


# ---------------------------------------------------------------------------
# Entry points (same names as the C ABI)
# ---------------------------------------------------------------------------

def opt2s_step(tl: TensorList, hyper: Hyper, step: int, stream=None) -> None:
    """One step of the whole collection in one launch (on torch's current
    stream unless ``stream`` is given)."""
    check(lib().opt2s_step(ctypes.byref(tl.desc), ctypes.byref(hyper), int(step),
                           _stream_handle(stream)), "opt2s_step")


def opt2s_step_noalloc(tl: TensorList, hyper: Hyper, step: int, stream=None) -> None:
    """opt2s_step for callers that cannot let the library allocate device
    memory (their runtime owns every byte through its own pool, or their
    footprint is fixed at start-up): the launch table lives in a fixed
    3 MiB device array instead of memory from cudaMalloc.  Collections that
    need more than opt2s_noalloc_max_chunks() chunk records are rejected;
    calls that overlap on the GPU race on the shared table."""
    check(lib().opt2s_step_noalloc(ctypes.byref(tl.desc), ctypes.byref(hyper), int(step),
                                   _stream_handle(stream)), "opt2s_step_noalloc")


def opt2s_step_max_unorm(tl: TensorList, hyper: Hyper, max_unorm: float, step: int,
                         stream=None) -> None:
    """opt2s_step with each tensor's update norm bounded by max_unorm times
    its weight norm (max_unorm > 0); four launches on `stream`."""
    check(lib().opt2s_step_max_unorm(ctypes.byref(tl.desc), ctypes.byref(hyper),
                                     float(max_unorm), int(step), _stream_handle(stream)),
          "opt2s_step_max_unorm")


def opt2s_step_lamb(tl: TensorList, hyper: Hyper, step: int, stream=None) -> None:
    """The LAMB step (You et al. 2020, Algorithm 2; Adam moments): per tensor,
    the Adam direction plus weight_decay * param, scaled by the trust ratio
    ||param|| / ||direction||; four launches on `stream`."""
    check(lib().opt2s_step_lamb(ctypes.byref(tl.desc), ctypes.byref(hyper), int(step),
                                _stream_handle(stream)), "opt2s_step_lamb")


def opt2s_step_8bit(tl: "TensorList8", hyper: Hyper, step: int, stream=None) -> None:
    """One step of a collection with 8-bit blockwise state (small tensors
    with fp32 state in the same launch)."""
    check(lib().opt2s_step_8bit(ctypes.byref(tl.desc), ctypes.byref(hyper), int(step),
                                _stream_handle(stream)), "opt2s_step_8bit")


def state_bits_for(numel: int, min_8bit_size: int = MIN_8BIT_SIZE) -> int:
    """8 when a tensor of numel elements keeps 8-bit state, else 32."""
    return int(lib().opt2s_8bit_state_bits(int(numel), int(min_8bit_size)))


def noalloc_max_chunks() -> int:
    return int(lib().opt2s_noalloc_max_chunks())


class Plan:
    """opt2s_plan_create / opt2s_plan_step / opt2s_plan_destroy."""

    def __init__(self, tl: TensorList, algo: str):
        self._h = ctypes.c_void_p()
        self._L = lib()   # a plan belongs to the library that made it
        self.tl = tl  # keep the descriptor alive with the plan
        check(self._L.opt2s_plan_create(ctypes.byref(tl.desc), ALGOS[algo],
                                        ctypes.byref(self._h)), "opt2s_plan_create", self._L)

    @property
    def num_chunks(self) -> int:
        return int(self._L.opt2s_plan_num_chunks(self._h))

    def step(self, hyper: Hyper, step: int, stream=None) -> None:
        check(self._L.opt2s_plan_step(self._h, ctypes.byref(hyper), int(step),
                                      _stream_handle(stream)), "opt2s_plan_step", self._L)

    def step_table(self, skip_zeros: bool, d_table: int, table_len: int, d_index: int,
                   stream=None) -> None:
        """opt2s_plan_step_table: the scalars come from d_table[*d_index]
        (device pointers), which the call then advances; capturable."""
        check(self._L.opt2s_plan_step_table(self._h, int(bool(skip_zeros)), d_table, int(table_len),
                                            d_index, _stream_handle(stream)), "opt2s_plan_step_table", self._L)

    def close(self) -> None:
        if self._h:
            check(self._L.opt2s_plan_destroy(self._h), "opt2s_plan_destroy", self._L)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def fill_step_scalars(hyper: Hyper, first_step: int, count: int) -> bytes:
    """opt2s_fill_step_scalars: the raw table of `count` steps (80 bytes each),
    ready to be copied to device memory."""
    arr = (opt2s_step_scalars * max(count, 1))()
    check(lib().opt2s_fill_step_scalars(ctypes.byref(hyper), int(first_step), int(count),
                                        ctypes.cast(arr, ctypes.c_void_p)), "opt2s_fill_step_scalars")
    return bytes(arr)[:count * ctypes.sizeof(opt2s_step_scalars)]


def opt2s_shard_range(numel: int, world: int, rank: int) -> tuple:
    """(start, length) of rank's shard of a flat buffer of numel elements."""
    a, n = ctypes.c_int64(), ctypes.c_int64()
    check(lib().opt2s_shard_range(int(numel), int(world), int(rank), ctypes.byref(a),
                                  ctypes.byref(n)), "opt2s_shard_range")
    return a.value, n.value


def make_shard_desc(world: int, rank: int, numel: int, dtype: int, params, grads,
                    state1, state2) -> opt2s_shard_desc:
    d = opt2s_shard_desc()
    d.world, d.rank, d.numel, d.dtype, d.reserved = world, rank, numel, dtype, 0
    for q in range(world):
        d.params[q] = _ptr(params[q])
        d.grads[q] = _ptr(grads[q])
    d.state1 = _ptr(state1) if state1 is not None else None
    d.state2 = _ptr(state2) if state2 is not None else None
    return d


def opt2s_shard_step(desc: opt2s_shard_desc, hyper: Hyper, step: int, stream=None) -> None:
    check(lib().opt2s_shard_step(ctypes.byref(desc), ctypes.byref(hyper), int(step),
                                 _stream_handle(stream)), "opt2s_shard_step")


def ipc_export(ptr) -> tuple:
    """(handle bytes, offset) of the device allocation holding ``ptr`` (an
    int address or a tensor), for another process's ipc_open."""
    h = opt2s_ipc_handle()
    off = ctypes.c_int64()
    check(lib().opt2s_ipc_export(_ptr(ptr), ctypes.byref(h), ctypes.byref(off)), "opt2s_ipc_export")
    return bytes(h.bytes), int(off.value)


def ipc_open(handle: bytes, offset: int) -> tuple:
    """Map another process's exported allocation: (base, address of its
    buffer).  Unmap with ipc_close(base)."""
    h = opt2s_ipc_handle()
    ctypes.memmove(h.bytes, handle, 64)
    base, ptr = ctypes.c_void_p(), ctypes.c_void_p()
    check(lib().opt2s_ipc_open(ctypes.byref(h), int(offset), ctypes.byref(base), ctypes.byref(ptr)),
          "opt2s_ipc_open")
    return int(base.value), int(ptr.value)


def ipc_close(base: int) -> None:
    check(lib().opt2s_ipc_close(int(base)), "opt2s_ipc_close")


def opt2s_release_cache() -> None:
    check(lib().opt2s_release_cache(), "opt2s_release_cache")


# ---------------------------------------------------------------------------
# Validation scaffolding (include/opt2s_testing.h) -- tests only.  The forcing
# knobs, the fault injection and the division check need testing_library().
# ---------------------------------------------------------------------------

def testing_build_chunks(tl: TensorList, algo: str, chunk_elems: int = 0) -> list:
    L = lib()
    n = ctypes.c_int64()
    check(L.opt2s_testing_build_chunks(ctypes.byref(tl.desc), ALGOS[algo], chunk_elems,
                                       None, 0, ctypes.byref(n)), "build_chunks")
    arr = (opt2s_testing_chunk * max(n.value, 1))()
    check(L.opt2s_testing_build_chunks(ctypes.byref(tl.desc), ALGOS[algo], chunk_elems,
                                       arr, n.value, ctypes.byref(n)), "build_chunks")
    return [(c.tensor, c.start, c.len, c.dtype) for c in arr[:n.value]]


def testing_unorm_tables(tl: TensorList, algo: str, chunk_elems: int = 0) -> dict:
    """The host tables of the bounded-update-norm step for `tl` (see
    opt2s_testing.h): block count, group ranges, first group per tensor and
    each chunk's tensor."""
    L = lib()
    counts = (ctypes.c_int64 * 3)()
    null = ctypes.POINTER(ctypes.c_uint32)()
    check(L.opt2s_testing_unorm_tables(ctypes.byref(tl.desc), ALGOS[algo], int(chunk_elems),
                                       null, null, null, counts), "testing_unorm_tables")
    ranges = (ctypes.c_uint32 * max(1, 2 * counts[1]))()
    first = (ctypes.c_uint32 * (tl.desc.count + 1))()
    chunks = (ctypes.c_uint32 * max(1, counts[2]))()
    check(L.opt2s_testing_unorm_tables(ctypes.byref(tl.desc), ALGOS[algo], int(chunk_elems),
                                       ranges, first, chunks, counts), "testing_unorm_tables")
    return {"nblocks": counts[0], "ranges": list(ranges[:2 * counts[1]]),
            "first_group": list(first), "chunk_tensor": list(chunks[:counts[2]])}


def testing_validate(tl: TensorList, hyper: Hyper, step: int) -> int:
    return lib().opt2s_testing_validate(ctypes.byref(tl.desc), ctypes.byref(hyper), int(step))


def testing_set_chunk_elems(n: int) -> int:
    return int(_testing_lib().opt2s_testing_set_chunk_elems(int(n)))


def testing_max_block_threads(algo: str, skip_zeros: bool) -> int:
    r = int(lib().opt2s_testing_max_block_threads(ALGOS[algo], int(bool(skip_zeros))))
    if r < 0:
        check(r, "testing_max_block_threads")
    return r


def testing_check_division(seed: int, n: int, mode: int) -> int:
    """Mismatches between the kernel's constant division and __fdiv_rn."""
    out = ctypes.c_int64()
    check(_testing_lib().opt2s_testing_check_division(seed, n, mode, ctypes.byref(out)),
          "check_division")
    return int(out.value)


def testing_choose_chunk_elems(tl: TensorList, resident_warps: int) -> int:
    return int(lib().opt2s_testing_choose_chunk_elems(ctypes.byref(tl.desc), int(resident_warps)))


def testing_fail_allocs(count: int) -> None:
    check(_testing_lib().opt2s_testing_fail_allocs(int(count)), "testing_fail_allocs")


QUANT_TABLE_WORDS = 512 + 3 * 26 * 128


def testing_quant_tables():
    """The 8-bit step's quantization tables as the library builds them:
    (signed map, unsigned map, signed slices x >= 0, x < 0, unsigned slices)."""
    import numpy as np
    buf = (ctypes.c_uint32 * QUANT_TABLE_WORDS)()
    check(lib().opt2s_testing_quant_tables(buf, QUANT_TABLE_WORDS), "testing_quant_tables")
    a = np.frombuffer(bytes(buf), np.uint32).copy()
    n = 26 * 128
    return (a[:256].view(np.float32), a[256:512].view(np.float32), a[512:512 + n],
            a[512 + n:512 + 2 * n], a[512 + 2 * n:])


def launch_count() -> int:
    """Kernels launched by libopt2s.so so far in this process."""
    return int(lib().opt2s_testing_launch_count())


def testing_set_launch(block_threads: int = 0, max_blocks: int = 0) -> None:
    check(_testing_lib().opt2s_testing_set_launch(int(block_threads), int(max_blocks)), "set_launch")
