"""Host-side checks of the C-ABI library; none of these launches a kernel.

* the shared library loads and exports every function include/lmoe.h declares;
* argument validation happens on the host, before any CUDA call, and returns
  the documented status codes;
* the Python binding exposes the same names.
"""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lmoe.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:int|const char \*)\s*(lmoe_\w+)\s*\(", text, re.M)))


@pytest.fixture(scope="module")
def lib():
    from latent_mixture_experts_top_b200 import build
    path = build.build()
    return C.CDLL(path)


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("lmoe_create", "lmoe_load_weights", "lmoe_route", "lmoe_forward",
              "lmoe_destroy"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in _declared():
        assert hasattr(lib, n), f"{n} declared in lmoe.h but not exported"


def test_binding_has_the_same_names(lib):
    from latent_mixture_experts_top_b200 import lmoe
    for n in _declared():
        assert callable(getattr(lmoe, n)), n
    assert set(lmoe.EXPORTED) >= set(_declared())


def test_binding_status_names_match_the_header():
    from latent_mixture_experts_top_b200 import lmoe
    codes = {int(v): k for k, v in re.findall(r"(LMOE_(?:OK|ERR_\w+))\s*=\s*(-?\d+)",
                                              open(HEADER).read())}
    assert codes == lmoe.STATUS


def _cfg(**kw):
    from latent_mixture_experts_top_b200 import lmoe
    base = dict(d=256, m=256, n_experts=8, top_k=2, alpha=2, n_shared=1, m_shared=256,
                variant=lmoe.LMOE_ACC, dtype=lmoe.LMOE_F32, n_routed_override=0,
                top_k_override=0, has_router_bias=0, max_tokens=64)
    base.update(kw)
    return lmoe.lmoe_config(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(d=0), -1), (dict(alpha=3), -1), (dict(alpha=0), -1), (dict(m=0), -1),
    (dict(top_k_override=17), -1), (dict(top_k=0), -1), (dict(variant=7), -1),
    (dict(dtype=5), -1), (dict(max_tokens=0), -1), (dict(n_shared=1, m_shared=0), -1),
    (dict(n_routed_override=2048, top_k_override=4), -7),
    (dict(dtype=1), -7),  # bf16 tiles need d, l multiples of 64 and m multiple of 128 ...
    # expert parallelism: N' = 16 experts over 3 ranks, a rank outside the
    # world, a negative world, and the fp32 mode (bf16 only)
    (dict(dtype=1, ep_world=3, ep_rank=0), -1), (dict(dtype=1, ep_world=2, ep_rank=2), -1),
    (dict(ep_world=-1), -1), (dict(ep_world=2, ep_rank=1), -7),
    # routed-expert formats: unknown; NVFP4 in the fp32 mode; NVFP4 with
    # l = 64 (quantised experts need l and m multiples of 128)
    (dict(weight_format=3), -1), (dict(weight_format=2), -7),
    (dict(dtype=1, weight_format=2, alpha=4), -7),
])
def test_create_rejects_bad_configs_on_host(lib, kw, code):
    from latent_mixture_experts_top_b200 import lmoe
    cfg = _cfg(**kw)
    if kw == dict(dtype=1):
        cfg.d, cfg.alpha, cfg.m, cfg.n_experts = 96, 1, 100, 8  # unsupported by the tiling
    h = C.c_void_p()
    rc = lib.lmoe_create(C.byref(cfg), C.byref(h))
    assert rc == code, lmoe.lmoe_strerror(rc)
    assert h.value is None


def test_null_arguments(lib):
    h = C.c_void_p()
    assert lib.lmoe_create(None, C.byref(h)) == -2
    assert lib.lmoe_create(C.byref(_cfg()), None) == -2
    assert lib.lmoe_forward(None, None, None, 0, None) == -2
    assert lib.lmoe_route(None, None, 0, None, None, None, None, None) == -2
    assert lib.lmoe_load_weights(None, None, None) == -2
    assert lib.lmoe_get_dims(None, None, None, None) == -2
    assert lib.lmoe_destroy(None) == 0
    assert lib.lmoe_ep_dispatch(None, None, 0, None, None, None) == -2
    assert lib.lmoe_ep_experts(None, None, None, 0, None, None) == -2
    assert lib.lmoe_ep_combine(None, None, None, 0, None) == -2
    assert lib.lmoe_forward_host_batches(None, 0, None, None, 0, None) == -2


def test_strerror_names_every_code(lib):
    lib.lmoe_strerror.restype = C.c_char_p
    seen = set()
    for code in range(0, -10, -1):
        s = lib.lmoe_strerror(code).decode()
        assert s and s != "unknown status"
        seen.add(s)
    assert len(seen) == 10
    assert lib.lmoe_strerror(-99).decode() == "unknown status"


def test_derived_sizes_follow_the_readme_variants():
    """N' = alpha N; K' = alpha K (acc) or K (eff); overrides win (README "Usage")."""
    from latent_mixture_experts_top_b200 import configs
    c = configs.README_ACC
    assert (c.l, c.n_routed, c.k_active) == (512, 256, 24)
    assert configs.README_EFF.k_active == 6
    assert (configs.PREFILL.l, configs.PREFILL.n_routed, configs.PREFILL.k_active) == (1024, 512, 22)
    assert (configs.TINY_F32.l, configs.TINY_F32.n_routed, configs.TINY_F32.k_active) == (128, 16, 4)
