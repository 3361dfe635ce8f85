"""ctypes binding of libaurora_muon.so (include/aurora_muon.h).

Argument marshalling only: every step of the optimizer runs in the library's
CUDA kernels.  The functions accept torch CUDA tensors (contiguous, 16-byte
aligned) and pass their device pointers plus the current CUDA stream.
The library must have been built (``python -m
aurora_orthogonalised_optimizer_b200.build``); a missing library is an error,
there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import os
from typing import List, Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libaurora_muon.so")
# AURORA_MUON_CHECKED=1 loads the bounds-checked build of the same library
# (every kernel's global accesses tested against their buffers' extents).
CHECKED_LIB_PATH = os.path.join(HERE, "libaurora_muon_checked.so")


def lib_path() -> str:
    return CHECKED_LIB_PATH if os.environ.get("AURORA_MUON_CHECKED", "0") == "1" else LIB_PATH

(MUON_OK, MUON_ERR_INVALID_ARG, MUON_ERR_UNSUPPORTED, MUON_ERR_WORKSPACE, MUON_ERR_CUDA, MUON_ERR_TIMEOUT,
 MUON_ERR_BOUNDS) = range(7)
MUON_F32, MUON_BF16 = 0, 1
MUON_GEMM_BF16, MUON_GEMM_FP32, MUON_GEMM_BF16_SIMT = 0, 1, 2

EXPORTS = ["muon_config_default", "muon_workspace_size", "muon_step", "ns_polar", "aurora_polar",
           "opnorm_normalize", "uw_floor_apply", "muon_last_device_status", "muon_status_string",
           "muon_profile_enable", "muon_profile_read", "opnorm_normalize_noalloc",
           "adamw_config_default", "adamw_step", "muon_selftest_wait_timeout", "muon_build_checked",
           "muon_last_check_line", "muon_selftest_bounds_check"]


class MuonShape(C.Structure):
    _fields_ = [("rows", C.c_int64), ("cols", C.c_int64)]


class MuonConfig(C.Structure):
    _fields_ = [
        ("lr", C.c_float), ("mu", C.c_float), ("nesterov", C.c_int),
        ("ns_steps", C.c_int), ("ns_a", C.c_float), ("ns_b", C.c_float), ("ns_c", C.c_float),
        ("ns_eps", C.c_float),
        ("aurora", C.c_int), ("pp_iterations", C.c_int), ("pp_beta", C.c_float), ("pp_eps", C.c_float),
        ("contra", C.c_float), ("power_iters", C.c_int),
        ("target_uw", C.c_float), ("weight_decay", C.c_float),
        ("gemm_mode", C.c_int), ("param_dtype", C.c_int), ("grad_dtype", C.c_int),
    ]


class AdamWConfig(C.Structure):
    _fields_ = [("lr", C.c_float), ("beta1", C.c_float), ("beta2", C.c_float), ("eps", C.c_float),
                ("weight_decay", C.c_float), ("step", C.c_int), ("param_dtype", C.c_int),
                ("grad_dtype", C.c_int)]


class MuonProfileEntry(C.Structure):
    _fields_ = [("name", C.c_char * 32), ("launches", C.c_int64), ("ms", C.c_double), ("flops", C.c_double),
                ("bytes", C.c_double)]


class MuonError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


_lib = None


def load():
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    path = lib_path()
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m aurora_orthogonalised_optimizer_b200.build`")
    lib = C.CDLL(path)
    P = C.c_void_p
    PP = C.POINTER(C.c_void_p)
    lib.muon_config_default.argtypes = [C.POINTER(MuonConfig)]
    lib.muon_config_default.restype = None
    lib.muon_workspace_size.argtypes = [C.POINTER(MuonConfig), C.c_int, C.POINTER(MuonShape)]
    lib.muon_workspace_size.restype = C.c_size_t
    lib.muon_step.argtypes = [C.POINTER(MuonConfig), C.c_int, C.POINTER(MuonShape), PP, PP, PP, PP,
                              P, C.c_size_t, P]
    lib.muon_step.restype = C.c_int
    for name in ("ns_polar", "aurora_polar"):
        f = getattr(lib, name)
        f.argtypes = [C.POINTER(MuonConfig), C.c_int, C.POINTER(MuonShape), PP, C.c_int, PP, P, C.c_size_t, P]
        f.restype = C.c_int
    lib.opnorm_normalize.argtypes = [C.POINTER(MuonConfig), C.c_int, C.POINTER(MuonShape), PP, C.c_int, PP,
                                     P, P, C.c_size_t, P]
    lib.opnorm_normalize.restype = C.c_int
    lib.opnorm_normalize_noalloc.argtypes = [C.POINTER(MuonConfig), C.c_int, C.POINTER(MuonShape), PP, C.c_int,
                                             PP, P, P]
    lib.opnorm_normalize_noalloc.restype = C.c_int
    lib.uw_floor_apply.argtypes = [C.POINTER(MuonConfig), C.c_int, C.POINTER(MuonShape), PP, PP, P,
                                   C.c_size_t, P]
    lib.uw_floor_apply.restype = C.c_int
    lib.muon_selftest_wait_timeout.argtypes = [C.c_longlong, P]
    lib.muon_selftest_wait_timeout.restype = C.c_int
    lib.muon_last_device_status.argtypes = [P]
    lib.muon_last_device_status.restype = C.c_int
    lib.muon_build_checked.argtypes = []
    lib.muon_build_checked.restype = C.c_int
    lib.muon_last_check_line.argtypes = []
    lib.muon_last_check_line.restype = C.c_int
    lib.muon_selftest_bounds_check.argtypes = [P]
    lib.muon_selftest_bounds_check.restype = C.c_int
    lib.muon_status_string.argtypes = [C.c_int]
    lib.muon_status_string.restype = C.c_char_p
    lib.adamw_config_default.argtypes = [C.POINTER(AdamWConfig)]
    lib.adamw_config_default.restype = None
    lib.adamw_step.argtypes = [C.POINTER(AdamWConfig), C.c_int, C.POINTER(C.c_int64), C.POINTER(C.c_float), PP, PP,
                               PP, PP, P]
    lib.adamw_step.restype = C.c_int
    lib.muon_profile_enable.argtypes = [C.c_int]
    lib.muon_profile_enable.restype = None
    lib.muon_profile_read.argtypes = [C.POINTER(MuonProfileEntry), C.c_int]
    lib.muon_profile_read.restype = C.c_int
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().muon_status_string(int(code)).decode()


# ---------------------------------------------------------------- config
@dataclasses.dataclass
class Config:
    """Python mirror of muon_config.  Defaults are the library defaults."""
    lr: float = 0.0375
    mu: float = 0.95
    nesterov: bool = True
    ns_steps: int = 12
    ns_a: float = 2.0
    ns_b: float = -1.5
    ns_c: float = 0.5
    ns_eps: float = 1e-7
    aurora: bool = True
    pp_iterations: int = 2
    pp_beta: float = 0.5
    pp_eps: float = 1e-7
    contra: float = 0.4
    power_iters: int = 5
    target_uw: float = 0.35
    weight_decay: float = 0.0
    gemm_mode: int = MUON_GEMM_BF16
    param_dtype: int = MUON_BF16
    grad_dtype: int = MUON_BF16

    @classmethod
    def from_step_config(cls, sc, **kw) -> "Config":
        """Copy the hyper-parameters of any object with the same field names."""
        vals = {f.name: getattr(sc, f.name) for f in dataclasses.fields(cls) if hasattr(sc, f.name)}
        vals.update(kw)
        return cls(**vals)

    def to_c(self) -> MuonConfig:
        c = MuonConfig()
        for f in dataclasses.fields(self):
            v = getattr(self, f.name)
            setattr(c, f.name, int(v) if isinstance(v, bool) else v)
        return c


def library_default_config() -> MuonConfig:
    c = MuonConfig()
    load().muon_config_default(C.byref(c))
    return c


def dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return MUON_BF16
    if t.dtype == torch.float32:
        return MUON_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


# ---------------------------------------------------------------- marshalling
def _shapes(shapes) -> C.Array:
    arr = (MuonShape * max(1, len(shapes)))()
    for i, (m, n) in enumerate(shapes):
        arr[i].rows, arr[i].cols = int(m), int(n)
    return arr


def _ptrs(ts: Optional[Sequence], n: int):
    if ts is None:
        return None
    arr = (C.c_void_p * max(1, n))()
    for i, t in enumerate(ts):
        arr[i] = None if t is None else int(t.data_ptr() if hasattr(t, "data_ptr") else t)
    return arr


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return int(stream.cuda_stream if hasattr(stream, "cuda_stream") else stream)


def _check_tensor(t, name):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def workspace_size(cfg: Config, shapes) -> int:
    return int(load().muon_workspace_size(C.byref(cfg.to_c()), len(shapes), _shapes(shapes)))


def make_workspace(cfg: Config, shapes, device=None):
    import torch
    n = workspace_size(cfg, shapes)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device or "cuda")


def _ws(ws):
    if ws is None:
        return None, 0
    return int(ws.data_ptr()), int(ws.numel() * ws.element_size())


def _raise(code, where):
    if code != MUON_OK:
        raise MuonError(code, where)


def muon_step(cfg: Config, params: List, grads: List, momentum: List, update_out: Optional[List] = None,
              workspace=None, stream=None, check: bool = True) -> int:
    n = len(params)
    shapes = [tuple(p.shape) for p in params]
    wp, wb = _ws(workspace)
    code = load().muon_step(C.byref(cfg.to_c()), n, _shapes(shapes), _ptrs(params, n), _ptrs(grads, n),
                            _ptrs(momentum, n), _ptrs(update_out, n), wp, wb, _stream(stream))
    if check:
        _raise(code, "muon_step")
    return code


def ns_polar(cfg: Config, inputs: List, outputs: List, workspace=None, stream=None, aurora: bool = False,
             check: bool = True) -> int:
    n = len(inputs)
    shapes = [tuple(t.shape) for t in inputs]
    dt = dtype_code(inputs[0]) if n else MUON_F32
    wp, wb = _ws(workspace)
    f = load().aurora_polar if aurora else load().ns_polar
    code = f(C.byref(cfg.to_c()), n, _shapes(shapes), _ptrs(inputs, n), dt, _ptrs(outputs, n), wp, wb,
             _stream(stream))
    if check:
        _raise(code, "aurora_polar" if aurora else "ns_polar")
    return code


def aurora_polar(cfg: Config, inputs: List, outputs: List, workspace=None, stream=None, check: bool = True):
    return ns_polar(cfg, inputs, outputs, workspace, stream, aurora=True, check=check)


def opnorm_normalize(cfg: Config, inputs: List, outputs: Optional[List], sigma_out=None, workspace=None,
                     stream=None, check: bool = True) -> int:
    n = len(inputs)
    shapes = [tuple(t.shape) for t in inputs]
    dt = dtype_code(inputs[0]) if n else MUON_F32
    wp, wb = _ws(workspace)
    code = load().opnorm_normalize(C.byref(cfg.to_c()), n, _shapes(shapes), _ptrs(inputs, n), dt,
                                   _ptrs(outputs, n), None if sigma_out is None else int(sigma_out.data_ptr()),
                                   wp, wb, _stream(stream))
    if check:
        _raise(code, "opnorm_normalize")
    return code


def opnorm_normalize_noalloc(cfg: Config, inputs: List, outputs: Optional[List], sigma_out=None, stream=None,
                             check: bool = True) -> int:
    """opnorm_normalize without a workspace, for callers that cannot allocate
    device memory at this point; scratch is the library's static 1 MiB array."""
    n = len(inputs)
    shapes = [tuple(t.shape) for t in inputs]
    dt = dtype_code(inputs[0]) if n else MUON_F32
    code = load().opnorm_normalize_noalloc(C.byref(cfg.to_c()), n, _shapes(shapes), _ptrs(inputs, n), dt,
                                           _ptrs(outputs, n),
                                           None if sigma_out is None else int(sigma_out.data_ptr()),
                                           _stream(stream))
    if check:
        _raise(code, "opnorm_normalize_noalloc")
    return code


def uw_floor_apply(cfg: Config, params: List, updates: List, workspace=None, stream=None,
                   check: bool = True) -> int:
    n = len(params)
    shapes = [tuple(t.shape) for t in params]
    wp, wb = _ws(workspace)
    code = load().uw_floor_apply(C.byref(cfg.to_c()), n, _shapes(shapes), _ptrs(params, n),
                                 _ptrs(updates, n), wp, wb, _stream(stream))
    if check:
        _raise(code, "uw_floor_apply")
    return code


def selftest_wait_timeout(max_cycles: int = 1_000_000, stream=None) -> int:
    """Run the bounded-wait timeout path once on the device (see the header)."""
    return int(load().muon_selftest_wait_timeout(int(max_cycles), _stream(stream)))


def last_device_status(stream=None) -> int:
    return int(load().muon_last_device_status(_stream(stream)))


def build_checked() -> bool:
    """True when the loaded library is the bounds-checked build."""
    return bool(load().muon_build_checked())


def last_check_line() -> int:
    """Where the first failed index test sits (checked build): file * 100000 + line, 0 if none."""
    return int(load().muon_last_check_line())


def selftest_bounds_check(stream=None) -> int:
    """Launch the index-test self-test (see the header)."""
    return int(load().muon_selftest_bounds_check(_stream(stream)))


def profile_enable(on: bool = True) -> None:
    load().muon_profile_enable(1 if on else 0)


def profile_read() -> dict:
    """Per-kernel-class totals recorded since profile_enable(True)."""
    arr = (MuonProfileEntry * 16)()
    n = load().muon_profile_read(arr, 16)
    if n < 0:
        raise MuonError(MUON_ERR_CUDA, "muon_profile_read")
    return {arr[i].name.decode(): {"launches": int(arr[i].launches), "ms": arr[i].ms, "flops": arr[i].flops,
                                   "bytes": arr[i].bytes} for i in range(n)}


def adamw_step(params: List, grads: List, exp_avg: List, exp_avg_sq: List, step: int, lr=0.01,
               beta1: float = 0.8, beta2: float = 0.95, eps: float = 1e-10, weight_decay: float = 0.0,
               stream=None, check: bool = True) -> int:
    """Fused AdamW over tensors (any shape, contiguous).  `lr` is a float or a
    per-tensor sequence.  Params/grads bf16 or fp32 (all alike); states fp32."""
    n = len(params)
    cfg = AdamWConfig()
    load().adamw_config_default(C.byref(cfg))
    per_tensor = not isinstance(lr, (int, float))
    cfg.lr = 0.0 if per_tensor else float(lr)
    cfg.beta1, cfg.beta2, cfg.eps, cfg.weight_decay, cfg.step = beta1, beta2, eps, weight_decay, int(step)
    if n:
        cfg.param_dtype = dtype_code(params[0])
        cfg.grad_dtype = dtype_code(grads[0])
    numels = (C.c_int64 * max(1, n))(*[int(p.numel()) for p in params])
    lrs = (C.c_float * max(1, n))(*[float(x) for x in lr]) if per_tensor else None
    code = load().adamw_step(C.byref(cfg), n, numels, lrs, _ptrs(params, n), _ptrs(grads, n), _ptrs(exp_avg, n),
                             _ptrs(exp_avg_sq, n), _stream(stream))
    if check:
        _raise(code, "adamw_step")
    return code
