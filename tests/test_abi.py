"""The C-ABI library loads and exports every symbol include/mp.h declares; host-side checks that run
before any CUDA call behave as documented. No compute call is made (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(mp_\w+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from atomistic_neighbor_list_b200 import build
    build.build()
    from atomistic_neighbor_list_b200 import mp
    return mp


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("mp_init", "mp_cfconv_fwd", "mp_attn_fwd", "mp_energy_forces", "mp_destroy",
                     "mp_strerror", "mp_neighbor_csr", "mp_neighbor_padded"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(lib.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(raw, n)]
    assert not missing, missing
    assert set(lib.EXPORTED) <= set(declared_functions())


def test_strerror_and_host_checks(lib):
    L = lib.lib
    assert L.mp_strerror(0) == b"ok"
    assert L.mp_strerror(-4) == b"CSR neighbor list is not symmetric"
    # null context / invalid configuration are rejected before any CUDA call
    assert L.mp_cfconv_fwd(None, 0, 1, 0, None, None, None, None, None, None) == -1
    assert L.mp_attn_fwd(None, 1, 1, None, None, None, None, None, None) == -1
    assert L.mp_energy_forces(None, 1, 0, None, None, None, None, None, 1, None, None, None) == -1
    cfg = lib.MpConfig(F=96, n_rbf=50, n_blocks=1, n_types=1, r_c=5.0, gamma=10.0, mu_max=5.0,
                       max_graphs=1)  # F=96 is not supported
    ctx = ctypes.c_void_p()
    w = lib.MpWeights()
    assert L.mp_init(ctypes.byref(ctx), ctypes.byref(cfg), ctypes.byref(w), None) == -1
    cfg.F, cfg.n_rbf = 128, 65  # too many radial functions
    assert L.mp_init(ctypes.byref(ctx), ctypes.byref(cfg), ctypes.byref(w), None) == -1
    cfg.n_rbf, cfg.n_heads, cfg.head_dim = 50, 16, 7  # heads x dim != F
    assert L.mp_init(ctypes.byref(ctx), ctypes.byref(cfg), ctypes.byref(w), None) == -1
    assert L.mp_neighbor_csr(-1, None, None, 1, 5.0, None, None, 0, None, None) == -1
    assert L.mp_neighbor_padded(4, None, None, 1, 5.0, 0, None, None, None) == -1
    assert L.mp_launch_count(None) == -1
    # the later entry points: a null context or a bad size is rejected on the host
    assert L.mp_attn_eq_fwd(None, 1, 1, None, None, None, None, None, None) == -1
    assert L.mp_attn_bwd(None, 1, 1, None, None, None, None, None, None, None, None) == -1
    assert L.mp_md_verlet(None, 1, 0, None, None, None, None, 0.01, 1, None, None, None, None, 1,
                          None, None, None) == -1
    n_edges = ctypes.c_longlong(0)
    assert L.mp_md_run(None, 1, None, None, None, None, 0.01, 1, None, None, 1, 0.5, 10, 0.25, 1,
                       None, None, 0, ctypes.byref(n_edges), None, None, None, None) == -1
    assert L.mp_spatial_order(-1, None, None, 1, 5.0, None, None) == -1
    assert L.mp_spatial_order(4, None, None, 1, 0.0, None, None) == -1


def test_struct_layout_matches_header(lib):
    assert ctypes.sizeof(lib.MpConfig) == 64
    assert ctypes.sizeof(lib.MpWeights) == 8 * (1 + 8 * 8 + 8) + 8
