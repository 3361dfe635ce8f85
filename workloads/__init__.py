"""Seeded synthetic inputs for the Muon / Aurora optimizer step.

This module is shared by the oracle-side tests and the CUDA-side tests and
bench.  It only draws random numbers, scales them and casts them to their
storage dtype; it holds none of the optimizer's arithmetic.

Every matrix is generated on its own from
``numpy.random.default_rng(SeedSequence([seed, matrix_index, step, stream]))``
with stream 0 = weights, 1 = gradient, 2 = per-matrix / per-row scales (drawn
once, step-independent).  Normals are drawn in float32, scaled in float32 and
rounded to the storage dtype (bfloat16 round-to-nearest-even, or kept as
float32).  bfloat16 arrays are carried as their raw ``uint16`` bit patterns.

Workload shapes follow the models the pages train: GPT-2 124M (12 layers,
d=768, MLP 4x) from the modded-nanogpt 2024-11-10 record write-up, and the
3.8B Llama-style model (28 layers, d=3072, GQA 24/8 heads, head_dim 128,
relu^2 MLP 12288) from "将 3.8B LLM 培训至 0.384 CORE，仅需 998 美元".
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor
from typing import List, Optional, Sequence, Tuple

import numpy as np

STREAM_W, STREAM_G, STREAM_SCALE = 0, 1, 2

F32, BF16 = "f32", "bf16"


# --------------------------------------------------------------------------
# storage casts (input side only)
# --------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round-to-nearest-even); return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 value of a stored array (bf16 bits or float32)."""
    if dtype == BF16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def store(x32: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16_bits(x32) if dtype == BF16 else np.ascontiguousarray(x32, np.float32)


# --------------------------------------------------------------------------
# hyper-parameters of a step (plain data; the library has its own struct)
# --------------------------------------------------------------------------
@dataclasses.dataclass
class StepConfig:
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


def aurora_stack(**kw) -> StepConfig:
    """Track-3 result #17 locked values: Aurora + Contra-Muon + u/w-floor."""
    return StepConfig(**kw)


def plain_muon(**kw) -> StepConfig:
    base = dict(aurora=False, contra=0.0, target_uw=0.0)
    base.update(kw)
    return StepConfig(**base)


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------
@dataclasses.dataclass
class Workload:
    name: str
    seed: int
    shapes: List[Tuple[int, int]]
    param_dtype: str
    grad_dtype: str
    w_std: Sequence[float]            # per matrix
    grad_kind: str                    # "unit", "matrix_scale", "row_lognormal"
    grad_base: float = 1.0
    grad_sigma: float = 0.0           # log-normal sigma for row scales
    cfg: StepConfig = dataclasses.field(default_factory=StepConfig)
    steps: int = 1

    @property
    def n(self) -> int:
        return len(self.shapes)

    def elements(self) -> int:
        return sum(m * n for m, n in self.shapes)


def gpt2_124m_shapes(layers: int = 12, d: int = 768) -> List[Tuple[int, int]]:
    out = []
    for _ in range(layers):
        out += [(d, d)] * 4 + [(4 * d, d), (d, 4 * d)]
    return out


def llama_3p8b_layer_shapes(d: int = 3072, kv: int = 1024, ff: int = 12288) -> List[Tuple[int, int]]:
    # q, k, v, o, fc, proj
    return [(d, d), (kv, d), (kv, d), (d, d), (ff, d), (d, ff)]


def llama_3p8b_shapes(layers: int = 28) -> List[Tuple[int, int]]:
    return llama_3p8b_layer_shapes() * layers


def fan_in_std(shapes):
    return [1.0 / math.sqrt(n) for (_, n) in shapes]


def single_aurora_256x128() -> Workload:
    s = [(256, 128)]
    return Workload("single_fp32_256x128_aurora", 0, s, F32, F32, [0.02], "unit",
                    cfg=aurora_stack(), steps=1)


def gpt2_124m_plain(steps: int = 5) -> Workload:
    s = gpt2_124m_shapes()
    return Workload("gpt2_124m_plain_muon", 1, s, BF16, BF16, fan_in_std(s), "matrix_scale",
                    cfg=plain_muon(lr=0.04, mu=0.90), steps=steps)


def aurora_shape_sweep(per_shape: int = 32) -> Workload:
    s = []
    for shp in [(1024, 4096), (4096, 1024), (2048, 2048), (768, 3072)]:
        s += [shp] * per_shape
    return Workload("aurora_sweep_4x32", 2, s, F32, F32, [0.02] * len(s), "row_lognormal",
                    grad_sigma=1.0, cfg=aurora_stack(), steps=1)


def llama_3p8b_plain(steps: int = 3, layers: int = 28) -> Workload:
    s = llama_3p8b_shapes(layers)
    return Workload("llama_3p8b_plain_muon", 3, s, BF16, BF16, fan_in_std(s), "unit",
                    grad_base=1e-3, cfg=plain_muon(lr=0.02, mu=0.95), steps=steps)


def llama_3p8b_aurora(steps: int = 3, layers: int = 28) -> Workload:
    s = llama_3p8b_shapes(layers)
    return Workload("llama_3p8b_aurora_stack", 4, s, BF16, BF16, fan_in_std(s), "row_lognormal",
                    grad_base=1e-3, grad_sigma=0.5, cfg=aurora_stack(), steps=steps)


WORKLOADS = {
    "single": single_aurora_256x128,
    "gpt2": gpt2_124m_plain,
    "sweep": aurora_shape_sweep,
    "llama_plain": llama_3p8b_plain,
    "llama_aurora": llama_3p8b_aurora,
}


def custom(name, seed, shapes, cfg, param_dtype=F32, grad_dtype=F32, w_std=0.02,
           grad_kind="unit", grad_base=1.0, grad_sigma=0.0, steps=1) -> Workload:
    if not isinstance(w_std, (list, tuple)):
        w_std = [w_std] * len(shapes)
    return Workload(name, seed, list(shapes), param_dtype, grad_dtype, list(w_std), grad_kind,
                    grad_base, grad_sigma, cfg, steps)


# --------------------------------------------------------------------------
# generation
# --------------------------------------------------------------------------
def _rng(seed: int, idx: int, step: int, stream: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, idx, step, stream]))


def weight(wl: Workload, idx: int) -> np.ndarray:
    m, n = wl.shapes[idx]
    x = _rng(wl.seed, idx, 0, STREAM_W).standard_normal((m, n), dtype=np.float32)
    x *= np.float32(wl.w_std[idx])
    return store(x, wl.param_dtype)


def grad(wl: Workload, idx: int, step: int = 0) -> np.ndarray:
    m, n = wl.shapes[idx]
    x = _rng(wl.seed, idx, step, STREAM_G).standard_normal((m, n), dtype=np.float32)
    srng = _rng(wl.seed, idx, 0, STREAM_SCALE)
    if wl.grad_kind == "matrix_scale":
        # 10^U(-4,-1): log-uniform per matrix in [1e-4, 1e-1]
        x *= np.float32(10.0 ** srng.uniform(-4.0, -1.0))
    elif wl.grad_kind == "row_lognormal":
        r = np.exp(wl.grad_sigma * srng.standard_normal(m)).astype(np.float32)
        x *= r[:, None]
    if wl.grad_base != 1.0:
        x *= np.float32(wl.grad_base)
    return store(x, wl.grad_dtype)


def momentum0(wl: Workload, idx: int) -> np.ndarray:
    m, n = wl.shapes[idx]
    return np.zeros((m, n), np.float32)


def generate(wl: Workload, indices: Optional[Sequence[int]] = None, step: int = 0,
             threads: int = 0):
    """Return (W list, G list, M list) for the given matrix indices."""
    idx = list(range(wl.n)) if indices is None else list(indices)

    def one(i):
        return weight(wl, i), grad(wl, i, step), momentum0(wl, i)

    if threads and len(idx) > 1:
        with ThreadPoolExecutor(threads) as ex:
            res = list(ex.map(one, idx))
    else:
        res = [one(i) for i in idx]
    return [r[0] for r in res], [r[1] for r in res], [r[2] for r in res]


def grads(wl: Workload, step: int, indices: Optional[Sequence[int]] = None, threads: int = 0):
    idx = list(range(wl.n)) if indices is None else list(indices)
    if threads and len(idx) > 1:
        with ThreadPoolExecutor(threads) as ex:
            return list(ex.map(lambda i: grad(wl, i, step), idx))
    return [grad(wl, i, step) for i in idx]


# --------------------------------------------------------------------------
# fast path for large workloads: the same float32 draws, cast to the storage
# dtype by torch on the CPU (round-to-nearest-even, identical values to
# f32_to_bf16_bits), returned as torch CPU tensors.
# --------------------------------------------------------------------------
def _draw_w32(wl: Workload, idx: int) -> np.ndarray:
    m, n = wl.shapes[idx]
    x = _rng(wl.seed, idx, 0, STREAM_W).standard_normal((m, n), dtype=np.float32)
    x *= np.float32(wl.w_std[idx])
    return x


def _draw_g32(wl: Workload, idx: int, step: int) -> np.ndarray:
    m, n = wl.shapes[idx]
    x = _rng(wl.seed, idx, step, STREAM_G).standard_normal((m, n), dtype=np.float32)
    srng = _rng(wl.seed, idx, 0, STREAM_SCALE)
    if wl.grad_kind == "matrix_scale":
        x *= np.float32(10.0 ** srng.uniform(-4.0, -1.0))
    elif wl.grad_kind == "row_lognormal":
        r = np.exp(wl.grad_sigma * srng.standard_normal(m)).astype(np.float32)
        x *= r[:, None]
    if wl.grad_base != 1.0:
        x *= np.float32(wl.grad_base)
    return x


def _to_torch(x32: np.ndarray, dtype: str):
    import torch
    t = torch.from_numpy(x32)
    return t.to(torch.bfloat16) if dtype == BF16 else t


def generate_torch(wl: Workload, indices: Optional[Sequence[int]] = None, step: int = 0, threads: int = 8,
                   want_w: bool = True, want_g: bool = True):
    """(W list, G list) as torch CPU tensors in their storage dtypes."""
    idx = list(range(wl.n)) if indices is None else list(indices)

    def one(i):
        w = _to_torch(_draw_w32(wl, i), wl.param_dtype) if want_w else None
        g = _to_torch(_draw_g32(wl, i, step), wl.grad_dtype) if want_g else None
        return w, g

    with ThreadPoolExecutor(max(1, threads)) as ex:
        res = list(ex.map(one, idx))
    return [r[0] for r in res], [r[1] for r in res]


# --------------------------------------------------------------------------
# the parameters the auxiliary AdamW steps (not the 2-D block matrices)
# --------------------------------------------------------------------------
@dataclasses.dataclass
class AuxWorkload:
    name: str
    seed: int
    shapes: List[Tuple[int, ...]]
    lrs: List[float]
    param_dtype: str = BF16
    grad_dtype: str = BF16
    beta1: float = 0.8
    beta2: float = 0.95
    eps: float = 1e-10
    weight_decay: float = 0.0

    @property
    def n(self) -> int:
        return len(self.shapes)

    def elements(self) -> int:
        return sum(int(np.prod(s)) for s in self.shapes)


def llama_3p8b_aux(layers: int = 28, vocab: int = 50304, d: int = 3072, kv: int = 1024,
                   value_tables: int = 14) -> AuxWorkload:
    """Token embedding (154.5M), untied LM head (154.5M), 14 value-embedding
    tables (721.2M) and per-layer 1-D gains of the 3.8B model; lrs as the
    Track 3 write-up sets them (embeddings 0.3, output projection 1/320,
    1-D parameters 0.01)."""
    shapes, lrs = [(vocab, d), (vocab, d)], [0.3, 1.0 / 320.0]
    shapes += [(vocab, kv)] * value_tables
    lrs += [0.3] * value_tables
    for _ in range(layers):
        shapes += [(d,), (d,), (1,), (1,)]       # two RMSNorm gains, two residual scalars
        lrs += [0.01] * 4
    return AuxWorkload("llama_3p8b_adamw_aux", 5, shapes, lrs)


def aux_param(wl: AuxWorkload, idx: int) -> np.ndarray:
    x = _rng(wl.seed, idx, 0, STREAM_W).standard_normal(wl.shapes[idx], dtype=np.float32)
    x *= np.float32(0.02)
    return store(x, wl.param_dtype)


def aux_grad(wl: AuxWorkload, idx: int, step: int = 0) -> np.ndarray:
    x = _rng(wl.seed, idx, step, STREAM_G).standard_normal(wl.shapes[idx], dtype=np.float32)
    x *= np.float32(1e-3)
    return store(x, wl.grad_dtype)
