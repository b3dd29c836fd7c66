"""The C-ABI library: it loads, exports every symbol include/lmoe.h declares,
and its host-side logic (configuration, validation, error paths that return
before any device work) behaves as documented.  No GPU needed."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

import latent_space_routed_b200 as lm


def _declared():
    with open(os.path.join(ROOT, "include", "lmoe.h")) as fh:
        src = fh.read()
    return sorted(set(re.findall(r"LMOE_API\s+[\w\s\*]*?\b(lmoe_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("lmoe_create", "lmoe_forward", "lmoe_destroy", "lmoe_workspace_size", "lmoe_config_from_base",
                 "lmoe_last_error", "lmoe_forward_host"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(lm.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    assert sorted(lm.EXPORTS) == sorted(_declared())


@pytest.mark.parametrize("variant,k", [("acc", 24), ("eff", 6)])
def test_config_from_base_readme_defaults(variant, k):
    """PyPI latent_moe README: d=2048, m=1408, N=64, K=6, alpha=4, n_shared=2;
    l = d/alpha, E = alpha N, k = K (eff) or alpha K (acc)."""
    c = lm.lmoe_config_from_base(2048, 1408, 64, 6, 4, 2, variant)
    assert (c.d, c.l, c.f, c.E, c.k, c.f_shared, c.n_shared) == (2048, 512, 1408, 256, k, 1408, 2)
    assert c.dtype == lm.LMOE_BF16 and c.act == lm.LMOE_ACT_SWIGLU
    assert abs(c.eps - 1e-6) < 1e-12


def test_config_from_base_standard_moe():
    """The base standard MoE the variants are derived from (cooking-agi
    LatentMoE page: experts at the model width, no projections): l = d,
    E = N, k = K."""
    c = lm.lmoe_config_from_base(2048, 1408, 64, 6, 4, 2, "std")
    assert (c.d, c.l, c.f, c.E, c.k, c.f_shared, c.standard) == (2048, 2048, 1408, 64, 6, 1408, 1)
    assert lm.lmoe_config_from_base(2048, 1408, 64, 6, 4, 2, "acc").standard == 0


@pytest.mark.parametrize("args", [(2048, 1408, 64, 6, 3, 2, "acc"), (2048, 1408, 64, 6, 4, 2, "big"),
                                  (0, 1408, 64, 6, 4, 2, "acc"), (2048, 1408, 2, 3, 1, 2, "eff")])
def test_config_from_base_rejects(args):
    with pytest.raises(lm.LmoeError) as ei:
        lm.lmoe_config_from_base(*args)
    assert ei.value.status == lm.LMOE_ERR_INVALID_ARG


def _cfg(**kw):
    base = dict(d=256, l=128, f=256, E=16, k=4, f_shared=256)
    base.update(kw)
    return lm.make_config(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(k=0), lm.LMOE_ERR_INVALID_ARG), (dict(k=17), lm.LMOE_ERR_INVALID_ARG),
    (dict(l=512), lm.LMOE_ERR_INVALID_ARG), (dict(n_shared=1), lm.LMOE_ERR_INVALID_ARG),
    (dict(d=0), lm.LMOE_ERR_INVALID_ARG), (dict(eps=-1.0), lm.LMOE_ERR_INVALID_ARG),
    (dict(dtype=7), lm.LMOE_ERR_INVALID_ARG), (dict(act=5), lm.LMOE_ERR_INVALID_ARG),
    (dict(d=200), lm.LMOE_ERR_UNSUPPORTED), (dict(E=2048, k=4), lm.LMOE_ERR_UNSUPPORTED),
    (dict(k=65, E=100), lm.LMOE_ERR_UNSUPPORTED),
    (dict(standard=1), lm.LMOE_ERR_INVALID_ARG), (dict(standard=2, l=256), lm.LMOE_ERR_INVALID_ARG),
])
def test_create_validates_before_touching_the_device(kw, status):
    """Constraints of "Stable LatentMoE" (two shared experts, 1 <= k <= E) and
    the cooking-agi latent_budget checks (l <= d) are rejected up front."""
    w = lm.lmoe_weights(*[1] * 10)   # never dereferenced: validation fails first
    h = ctypes.c_void_p()
    cfg = _cfg(**kw)
    st = lm._lib.lmoe_create(ctypes.byref(cfg), ctypes.byref(w), None, ctypes.byref(h))
    assert st == status, lm.lmoe_last_error()
    assert h.value is None
    assert lm.lmoe_last_error() != ""


def test_null_arguments():
    lib = lm._lib
    n = ctypes.c_size_t()
    assert lib.lmoe_workspace_size(None, 4, ctypes.byref(n)) == lm.LMOE_ERR_INVALID_ARG
    assert lib.lmoe_forward(None, None, 4, None, None, None, None, None, 0, None) == lm.LMOE_ERR_INVALID_ARG
    cfg = _cfg()
    h = ctypes.c_void_p()
    assert lib.lmoe_create(ctypes.byref(cfg), None, None, ctypes.byref(h)) == lm.LMOE_ERR_INVALID_ARG
    assert lib.lmoe_create(None, None, None, ctypes.byref(h)) == lm.LMOE_ERR_INVALID_ARG
    lib.lmoe_destroy(None)   # ignored


def test_missing_library_fails_loudly(tmp_path):
    """Without the built library the package refuses to import (no fallback)."""
    import shutil
    import subprocess
    import sys
    pkg = tmp_path / "latent_space_routed_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(os.path.dirname(lm.__file__), "__init__.py"), pkg / "__init__.py")
    r = subprocess.run([sys.executable, "-c", "import latent_space_routed_b200"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0
    assert "liblmoe.so is missing" in r.stderr


def test_product_never_reaches_the_oracle():
    """The package and its sources name neither the oracle nor a CPU path for the layer."""
    root = os.path.dirname(lm.__file__)
    for dirpath, _, files in os.walk(root):
        for name in files:
            if name.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, name)).read()
                assert "import oracle" not in text and "from oracle" not in text, name
                assert "lmoe_oracle" not in text, name

