"""The single-SM tensor-core GEMM variant (AURORA_MUON_TC_PAIR=0: 128 x 256
tiles, cta_group::1) against the oracle, full Aurora stack, in a child
process (the variant is chosen once per process).  It shares the kernel
source with the default SM-pair variant but has its own tile decomposition
of the symmetric kinds and its own slots for the fused <U,U>, <U,u>."""
import json
import os
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import json, sys
import numpy as np, torch
sys.path.insert(0, ROOT)
import workloads as WL, oracle.muon_oracle as O
from aurora_orthogonalised_optimizer_b200 import _abi as A
shapes = [(256, 128), (192, 320), (640, 384), (300, 300)]
wl = WL.custom("single_sm", 21, shapes, WL.aurora_stack(), WL.BF16, WL.BF16, w_std=0.05)
cfg = A.Config.from_step_config(wl.cfg, gemm_mode=A.MUON_GEMM_BF16, param_dtype=A.MUON_BF16, grad_dtype=A.MUON_BF16)
W, G, M = WL.generate(wl)
p = [torch.from_numpy(WL.bf16_bits_to_f32(w) if w.dtype == np.uint16 else w).to(torch.bfloat16).cuda() for w in W]
g = [torch.from_numpy(WL.bf16_bits_to_f32(x) if x.dtype == np.uint16 else x).to(torch.bfloat16).cuda() for x in G]
m = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in shapes]
v = [torch.empty(s, dtype=torch.float32, device="cuda") for s in shapes]
A.muon_step(cfg, p, g, m, v, A.make_workspace(cfg, shapes))
torch.cuda.synchronize()
out = {"status": int(A.last_device_status()), "err": []}
for k in range(len(shapes)):
    _, _, V = O.step(WL.to_f64(W[k], WL.BF16), WL.to_f64(G[k], WL.BF16), M[k].astype(np.float64), wl.cfg, WL.BF16)
    d = v[k].double().cpu().numpy()
    out["err"].append(float(np.linalg.norm(d - V) / np.linalg.norm(V)))
print(json.dumps(out))
'''.replace("ROOT", repr(ROOT))


def test_single_sm_variant_matches_oracle():
    env = dict(os.environ, AURORA_MUON_TC_PAIR="0")
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    out = json.loads(r.stdout.strip().splitlines()[-1])
    assert out["status"] == 0
    for e in out["err"]:
        assert e <= 3e-2, out["err"]


SYM_CHILD = r'''
import json, sys
import numpy as np, torch
sys.path.insert(0, ROOT)
import oracle.muon_oracle as O
from aurora_orthogonalised_optimizer_b200 import _abi as A
out = {"status": 0, "asym": [], "err": []}
for (s, k) in [(300, 200), (257, 40), (520, 520)]:
    for (a, b, c) in [(0.0, 1.0, 0.0), (0.0, 0.0, 1.0)]:
        cfg = A.Config(gemm_mode=A.MUON_GEMM_BF16, ns_steps=1, ns_a=a, ns_b=b, ns_c=c)
        X = np.concatenate([np.random.default_rng(31 + s).standard_normal((s, k)).astype(np.float32),
                            np.eye(s, dtype=np.float32)], axis=1)
        o = torch.empty(X.shape, dtype=torch.float32, device="cuda")
        A.ns_polar(cfg, [torch.from_numpy(X).cuda()], [o], A.make_workspace(cfg, [X.shape]))
        torch.cuda.synchronize()
        out["status"] |= int(A.last_device_status())
        got = o.double().cpu().numpy()[:, k:]
        want = O.newton_schulz(X.astype(np.float64), 1, a, b, c, 1e-7)[:, k:]
        out["asym"].append(int(np.count_nonzero(got != got.T)))
        out["err"].append(float(np.max(np.abs(got - want)) / np.max(np.abs(want))))
print(json.dumps(out))
'''.replace("ROOT", repr(ROOT))


def test_single_sm_variant_symmetric_blocks_exactly_symmetric():
    """The single-SM variant's own tiling of the Gram and square kinds (128 x
    256 tiles, so a tile's diagonal 32 x 32 blocks fall in its left or its
    right half): the symmetric product read back through X = [M | I] is
    exactly symmetric and close to float64 (see
    test_symmetric_gemm_blocks_exactly_symmetric)."""
    env = dict(os.environ, AURORA_MUON_TC_PAIR="0")
    r = subprocess.run([sys.executable, "-c", SYM_CHILD], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    out = json.loads(r.stdout.strip().splitlines()[-1])
    assert out["status"] == 0
    assert out["asym"] == [0] * len(out["asym"]), out["asym"]
    assert max(out["err"]) <= 1e-2, out["err"]
