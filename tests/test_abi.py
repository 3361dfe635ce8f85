"""Host-side checks of the C ABI: symbols, defaults, workspace sizing and
argument validation.  No call here reaches a kernel launch: every invalid
request is rejected on the host before anything is launched."""
import ctypes as C
import json
import os
import re

import pytest

from aurora_orthogonalised_optimizer_b200 import _abi as A

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLD = os.path.join(ROOT, "tests", "golden")


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(",
                                src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(A.EXPORTS) <= set(names)
    for name in names:
        assert hasattr(lib, name), name


def test_config_struct_layout_matches_header(lib):
    c = A.library_default_config()
    assert C.sizeof(A.MuonConfig) == 19 * 4
    g = json.load(open(os.path.join(GOLD, "page_constants.json")))
    assert c.ns_steps == g["ns_steps"]["value"]
    assert c.ns_a == pytest.approx(g["ns_a"]["value"])
    assert c.ns_b == pytest.approx(g["ns_b"]["value"])
    assert c.ns_c == pytest.approx(g["ns_c"]["value"])
    assert c.ns_eps == pytest.approx(g["ns_eps"]["value"])
    assert c.pp_iterations == g["pp_iterations"]["value"]
    assert c.pp_beta == pytest.approx(g["pp_beta"]["value"])
    assert c.contra == pytest.approx(g["contra"]["value"])
    assert c.power_iters == g["power_iters"]["value"]
    assert c.target_uw == pytest.approx(g["target_uw"]["value"])
    assert c.lr == pytest.approx(g["lr_aurora"]["value"])
    assert c.mu == pytest.approx(g["mu"]["value"])
    assert c.weight_decay == 0.0 and c.nesterov == 1 and c.aurora == 1
    # the Python mirror has the same defaults
    py = A.Config().to_c()
    for f, _ in A.MuonConfig._fields_:
        assert getattr(py, f) == pytest.approx(getattr(c, f)), f


def test_status_strings(lib):
    for code in range(6):
        assert A.status_string(code)
    assert A.status_string(A.MUON_ERR_WORKSPACE).startswith("workspace")


def test_workspace_size_properties(lib):
    cfg = A.Config()
    assert A.workspace_size(cfg, []) == 0
    a = A.workspace_size(cfg, [(256, 128)])
    b = A.workspace_size(cfg, [(256, 128), (128, 256)])
    c = A.workspace_size(A.Config(gemm_mode=A.MUON_GEMM_FP32), [(256, 128)])
    assert 0 < a < b
    assert c > a                       # fp32 NS buffers are twice as large
    big = A.workspace_size(cfg, [(12288, 3072)])
    # u, two X ping-pong buffers (bf16, s x l) + A, B (s x s)
    assert big >= 3 * 3072 * 12288 * 2 + 2 * 3072 * 3072 * 2


def _cfg(**kw):
    return A.Config(**kw).to_c()


FAKE = 0x7f0000000000  # aligned fake device address: never dereferenced (all calls below fail validation)


def _arr(*vals):
    a = (C.c_void_p * len(vals))()
    for i, v in enumerate(vals):
        a[i] = v
    return a


def _call_step(lib, cfg, shapes, params, grads, mom, ws=FAKE, ws_bytes=0):
    sh = A._shapes(shapes)
    return lib.muon_step(C.byref(cfg) if cfg is not None else None, len(shapes), sh, params, grads, mom, None,
                         ws, ws_bytes, None)


def test_validation_rejects_before_launch(lib):
    shapes = [(64, 32)]
    p, g, m = _arr(FAKE), _arr(FAKE + 4096), _arr(FAKE + 8192)
    assert _call_step(lib, None, shapes, p, g, m) == A.MUON_ERR_INVALID_ARG
    assert _call_step(lib, _cfg(weight_decay=0.1), shapes, p, g, m) == A.MUON_ERR_INVALID_ARG
    assert _call_step(lib, _cfg(ns_steps=0), shapes, p, g, m) == A.MUON_ERR_INVALID_ARG
    assert _call_step(lib, _cfg(pp_iterations=0), shapes, p, g, m) == A.MUON_ERR_INVALID_ARG
    assert _call_step(lib, _cfg(power_iters=0), shapes, p, g, m) == A.MUON_ERR_INVALID_ARG
    assert _call_step(lib, _cfg(gemm_mode=7), shapes, p, g, m) == A.MUON_ERR_INVALID_ARG
    assert _call_step(lib, _cfg(param_dtype=5), shapes, p, g, m) == A.MUON_ERR_INVALID_ARG
    assert _call_step(lib, _cfg(), [(0, 32)], p, g, m) == A.MUON_ERR_INVALID_ARG
    assert _call_step(lib, _cfg(), [(64, -1)], p, g, m) == A.MUON_ERR_INVALID_ARG
    assert _call_step(lib, _cfg(), shapes, _arr(None), g, m) == A.MUON_ERR_INVALID_ARG
    assert _call_step(lib, _cfg(), shapes, p, _arr(FAKE + 2), m) == A.MUON_ERR_INVALID_ARG   # misaligned
    assert _call_step(lib, _cfg(), shapes, p, g, None) == A.MUON_ERR_INVALID_ARG
    # workspace missing / too small
    assert _call_step(lib, _cfg(), shapes, p, g, m, ws=None, ws_bytes=1 << 30) == A.MUON_ERR_WORKSPACE
    need = A.workspace_size(A.Config(), shapes)
    assert _call_step(lib, _cfg(), shapes, p, g, m, ws=FAKE, ws_bytes=need - 1) == A.MUON_ERR_WORKSPACE
    # contra off: power_iters is not checked
    assert _call_step(lib, _cfg(contra=0.0, power_iters=0), shapes, p, g, m, ws=None) == A.MUON_ERR_WORKSPACE
    # n == 0 is a no-op
    assert lib.muon_step(C.byref(_cfg()), 0, None, None, None, None, None, None, 0, None) == A.MUON_OK


def test_other_entry_points_validate(lib):
    sh = A._shapes([(16, 8)])
    cfg = _cfg()
    x, y = _arr(FAKE), _arr(FAKE + 4096)
    assert lib.ns_polar(C.byref(cfg), 1, sh, x, 3, y, None, 0, None) == A.MUON_ERR_INVALID_ARG
    assert lib.ns_polar(C.byref(cfg), 1, sh, x, 0, None, None, 0, None) == A.MUON_ERR_INVALID_ARG
    assert lib.ns_polar(C.byref(cfg), 1, sh, x, 0, y, None, 0, None) == A.MUON_ERR_WORKSPACE
    assert lib.aurora_polar(C.byref(_cfg(pp_iterations=0)), 1, sh, x, 0, y, None, 0, None) == A.MUON_ERR_INVALID_ARG
    assert lib.opnorm_normalize(C.byref(_cfg(power_iters=0)), 1, sh, x, 0, y, None, None, 0, None) == \
        A.MUON_ERR_INVALID_ARG
    assert lib.opnorm_normalize(C.byref(cfg), 1, sh, x, 0, None, FAKE + 2, None, 0, None) == \
        A.MUON_ERR_INVALID_ARG
    assert lib.uw_floor_apply(None, 1, sh, x, y, None, 0, None) == A.MUON_ERR_INVALID_ARG
    assert lib.uw_floor_apply(C.byref(cfg), 1, sh, x, _arr(None), None, 0, None) == A.MUON_ERR_INVALID_ARG
    assert lib.uw_floor_apply(C.byref(cfg), 1, sh, x, y, None, 0, None) == A.MUON_ERR_WORKSPACE


def test_adamw_defaults_and_validation(lib):
    c = A.AdamWConfig()
    lib.adamw_config_default(C.byref(c))
    assert c.beta1 == pytest.approx(0.8) and c.beta2 == pytest.approx(0.95)
    assert c.eps == pytest.approx(1e-10) and c.weight_decay == 0.0 and c.step == 1
    n1 = (C.c_int64 * 1)(16)
    x = _arr(FAKE)
    def call(cfg, numels=n1, p=x, g=x, m=x, v=x):
        return lib.adamw_step(C.byref(cfg) if cfg is not None else None, 1, numels, None, p, g, m, v, None)
    assert call(None) == A.MUON_ERR_INVALID_ARG
    for field, bad in [("step", 0), ("beta1", 1.0), ("beta2", -0.1), ("eps", -1.0), ("weight_decay", -1.0),
                       ("param_dtype", 3)]:
        b = A.AdamWConfig()
        lib.adamw_config_default(C.byref(b))
        setattr(b, field, bad)
        assert call(b) == A.MUON_ERR_INVALID_ARG, field
    assert call(c, numels=(C.c_int64 * 1)(-1)) == A.MUON_ERR_INVALID_ARG
    assert call(c, m=_arr(FAKE + 4)) == A.MUON_ERR_INVALID_ARG          # misaligned
    assert call(c, g=_arr(None)) == A.MUON_ERR_INVALID_ARG
    assert lib.adamw_step(C.byref(c), 0, None, None, None, None, None, None, None) == A.MUON_OK


def test_size_limits_are_rejected_on_the_host(lib):
    p, g, m = _arr(FAKE), _arr(FAKE + 4096), _arr(FAKE + 8192)
    # the smaller side above 32768 is not supported; nothing is sized or launched
    assert _call_step(lib, _cfg(), [(40000, 40000)], p, g, m) == A.MUON_ERR_UNSUPPORTED
    assert A.workspace_size(A.Config(), [(40000, 40000)]) == 0
    assert _call_step(lib, _cfg(), [(1 << 32, 8)], p, g, m) == A.MUON_ERR_INVALID_ARG


def test_noalloc_entry_rejects_oversized_edges_on_the_host(lib):
    """rows or cols above 2^31 are refused before the scratch size is summed
    (near 2^62 the sum would wrap around and pass the 1 MiB check)."""
    cfg = A.Config()
    ptrs = (C.c_void_p * 1)(FAKE)
    for shape in [((1 << 62) - 64, 8), (8, (1 << 62) - 64), ((1 << 31) + 1, 1)]:
        code = lib.opnorm_normalize_noalloc(C.byref(cfg.to_c()), 1, A._shapes([shape]), ptrs, A.MUON_F32,
                                            None, None, None)
        assert code == A.MUON_ERR_INVALID_ARG, shape
    code = lib.opnorm_normalize_noalloc(C.byref(cfg.to_c()), 1, A._shapes([(1 << 31, 1 << 31)]), ptrs,
                                        A.MUON_F32, None, None, None)
    assert code == A.MUON_ERR_UNSUPPORTED          # inside the edge bound, beyond the scratch


def test_checked_library_exports_the_same_symbols():
    """The bounds-checked build (libaurora_muon_checked.so) loads on the host,
    exports every declared symbol and says it is the checked one."""
    path = A.CHECKED_LIB_PATH
    assert os.path.exists(path), "build it with build.py --checked"
    chk = C.CDLL(path)
    for name in declared_functions():
        assert hasattr(chk, name), name
    chk.muon_build_checked.restype = C.c_int
    assert chk.muon_build_checked() == 1
    plain = C.CDLL(A.LIB_PATH)
    plain.muon_build_checked.restype = C.c_int
    assert plain.muon_build_checked() == 0
    chk.muon_status_string.restype = C.c_char_p
    assert b"checked build" in chk.muon_status_string(A.MUON_ERR_BOUNDS)
