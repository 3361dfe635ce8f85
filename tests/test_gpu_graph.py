"""muon_step inside a CUDA graph: the entry point issues only kernel launches
and workspace memsets on the caller's stream (no allocation, no
synchronisation, no host read of device data), so a captured step replays to
the same bits as an eager one.
This is what lets a launch-bound caller (small matrices, ~125 launches per
step) replace the per-launch host cost with one graph launch."""
import pytest

import workloads as WL

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

from aurora_orthogonalised_optimizer_b200 import _abi as A  # noqa: E402


def _state(wl):
    W, G = WL.generate_torch(wl, None, 0)
    p = [w.cuda() for w in W]
    g = [x.cuda() for x in G]
    m = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in wl.shapes]
    return p, g, m


@pytest.mark.parametrize("stack", ["aurora", "plain"])
def test_captured_step_replays_bitwise(stack):
    shapes = [(768, 768), (3072, 768), (768, 3072), (256, 128), (200, 72)]
    sc = WL.aurora_stack() if stack == "aurora" else WL.plain_muon(lr=0.04, mu=0.9)
    wl = WL.custom("graph", 9, shapes, sc, WL.BF16, WL.BF16, w_std=0.03)
    cfg = A.Config.from_step_config(wl.cfg, gemm_mode=A.MUON_GEMM_BF16, param_dtype=A.MUON_BF16,
                                    grad_dtype=A.MUON_BF16)
    ws = A.make_workspace(cfg, shapes)

    # eager: two steps from the initial state
    p0, g0, m0 = _state(wl)
    pe, me = [t.clone() for t in p0], [t.clone() for t in m0]
    for _ in range(2):
        A.muon_step(cfg, pe, g0, me, None, ws)
    torch.cuda.synchronize()
    assert A.last_device_status() == A.MUON_OK

    # captured: warm up on a side stream (first-call set-up happens there), capture one step, replay twice
    pc, mc = [t.clone() for t in p0], [t.clone() for t in m0]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        pw, mw = [t.clone() for t in p0], [t.clone() for t in m0]
        A.muon_step(cfg, pw, g0, mw, None, ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        A.muon_step(cfg, pc, g0, mc, None, ws)
    # capture records the launches without running them: the state is still the initial one
    torch.cuda.synchronize()
    for a, b in zip(pc, p0):
        assert torch.equal(a, b)
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    assert A.last_device_status() == A.MUON_OK
    for a, b in zip(pc, pe):
        assert torch.equal(a, b)
    for a, b in zip(mc, me):
        assert torch.equal(a, b)
