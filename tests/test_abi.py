"""The C ABI without a GPU: the library builds, loads, exports every entry point
include/lamp.h declares, and rejects bad arguments on the host before any
CUDA call (so these checks run on a machine with no device)."""
import ctypes
import os
import re

import pytest

import mixed_precision_attention_ps_b200 as lamp
from mixed_precision_attention_ps_b200 import _native, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "lamp.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _native.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"LAMP_API\s+[\w\s\*]*?\b(lamp_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    assert {"lamp_attention", "lamp_attention_ex", "lamp_workspace_size", "lamp_last_error",
            "lamp_ps_round", "lamp_version", "lamp_args_size"} <= set(names)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert set(declared_symbols()) == set(_native.SIGNATURES)


def test_struct_layout_matches(lib):
    assert lamp.lamp_args_size() == ctypes.sizeof(_native.lamp_args) == 176
    assert lamp.lamp_gelu_args_size() == ctypes.sizeof(_native.lamp_gelu_args) == 112
    assert lamp.lamp_ln_args_size() == ctypes.sizeof(_native.lamp_ln_args) == 136
    assert lamp.lamp_version().startswith("lamp-b200")


FAKE = 1 << 20  # a 16-byte aligned non-null address; never dereferenced (checks fail first)


def call_ex(**kw):
    base = dict(dims=(1, 1, 128, 128, 64), Q=FAKE, K=FAKE, V=FAKE, out=FAKE, mu=4, tau=0.05,
                variant=lamp.LAMP_STRICT, causal=1)
    base.update(kw)
    return lamp.lamp_attention_ex(check=False, **base)


@pytest.mark.parametrize("kw,code,msg", [
    (dict(Q=None), lamp.LAMP_ERR_ARG, "non-NULL"),
    (dict(out=None), lamp.LAMP_ERR_ARG, "non-NULL"),
    (dict(mu=0), lamp.LAMP_ERR_ARG, "mu"),
    (dict(mu=24), lamp.LAMP_ERR_ARG, "mu"),
    (dict(tau=float("nan")), lamp.LAMP_ERR_ARG, "tau"),
    (dict(variant=3), lamp.LAMP_ERR_ARG, "variant"),
    (dict(variant=lamp.LAMP_GIVEN_MASK), lamp.LAMP_ERR_ARG, "mask_in"),
    (dict(causal=2), lamp.LAMP_ERR_ARG, "causal"),
    (dict(scale=-1.0), lamp.LAMP_ERR_ARG, "scale"),
    (dict(scale=float("inf")), lamp.LAMP_ERR_ARG, "scale"),
    (dict(dims=(0, 1, 128, 128, 64)), lamp.LAMP_ERR_ARG, "positive"),
    (dict(dims=(1, 1, 128, -1, 64)), lamp.LAMP_ERR_ARG, "positive"),
    (dict(dims=(1, 1, 128, 128, 96)), lamp.LAMP_ERR_UNSUPPORTED, "d must be"),
    (dict(Q=FAKE + 8), lamp.LAMP_ERR_UNSUPPORTED, "16-byte"),
    (dict(out_f32=FAKE + 4), lamp.LAMP_ERR_UNSUPPORTED, "aligned"),
    (dict(n_selected_out=FAKE + 4), lamp.LAMP_ERR_UNSUPPORTED, "aligned"),
    (dict(debug_stall=7), lamp.LAMP_ERR_ARG, "debug_stall"),
])
def test_argument_checks(lib, kw, code, msg):
    rc = call_ex(**kw)
    assert rc == code
    assert msg in lamp.lamp_last_error()


def test_basic_entry_rejects_given_mask_and_null_dims(lib):
    L = _native.load()
    assert L.lamp_attention(None, FAKE, FAKE, FAKE, FAKE, None, 4, 0.1, 0, 1, None) == lamp.LAMP_ERR_ARG
    rc = lamp.lamp_attention((1, 1, 8, 8, 64), FAKE, FAKE, FAKE, FAKE, None, 4, 0.1,
                             lamp.LAMP_GIVEN_MASK, 1, check=False)
    assert rc == lamp.LAMP_ERR_ARG and "lamp_attention_ex" in lamp.lamp_last_error()


def test_checked_call_raises_with_message(lib):
    with pytest.raises(lamp.LampError) as ei:
        lamp.lamp_attention_ex(dims=(1, 1, 8, 8, 64), Q=FAKE, K=FAKE, V=FAKE, out=FAKE, mu=99)
    assert ei.value.code == lamp.LAMP_ERR_ARG


def test_workspace_size_of_invalid_dims_is_zero(lib):
    assert lamp.lamp_workspace_size((1, 1, 0, 8, 64), 0) == 0
    assert lamp.lamp_workspace_size((1, 1, 8, 8, 80), 0) == 0
    assert lamp.lamp_workspace_size((1, 1, 8, 8, 64), 7) == 0


def test_ps_round_argument_checks(lib):
    assert lamp.lamp_ps_round(None, None, 0, 4, 0, check=False) == 0        # empty: nothing to do
    assert lamp.lamp_ps_round(None, None, 5, 4, 0, check=False) == lamp.LAMP_ERR_ARG
    assert lamp.lamp_ps_round(FAKE, FAKE, 5, 0, 0, check=False) == lamp.LAMP_ERR_ARG
    assert lamp.lamp_ps_round(FAKE, FAKE, 5, 4, 2, check=False) == lamp.LAMP_ERR_ARG


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(_native, "_lib", None)
    with pytest.raises(ImportError, match="no fallback"):
        _native.load(str(tmp_path / "liblamp.so"))


def call_gelu(**kw):
    base = dict(M=4, N=40, K=16, x=FAKE, W=FAKE, out=FAKE, mu=4, tau=1.0)
    base.update(kw)
    return lamp.lamp_linear_gelu(check=False, **base)


@pytest.mark.parametrize("kw,code,msg", [
    (dict(x=None), lamp.LAMP_ERR_ARG, "non-NULL"),
    (dict(out=None), lamp.LAMP_ERR_ARG, "non-NULL"),
    (dict(M=0), lamp.LAMP_ERR_ARG, "positive"),
    (dict(K=-8), lamp.LAMP_ERR_ARG, "positive"),
    (dict(mu=24), lamp.LAMP_ERR_ARG, "mu"),
    (dict(variant=lamp.LAMP_RELAXED), lamp.LAMP_ERR_ARG, "relaxed"),
    (dict(variant=5), lamp.LAMP_ERR_ARG, "variant"),
    (dict(tau=float("nan")), lamp.LAMP_ERR_ARG, "tau"),
    (dict(variant=lamp.LAMP_GIVEN_MASK), lamp.LAMP_ERR_ARG, "mask_in"),
    (dict(scale=float("inf")), lamp.LAMP_ERR_ARG, "scale"),
    (dict(K=12), lamp.LAMP_ERR_UNSUPPORTED, "multiple of 8"),
    (dict(M=65535 * 64 + 1), lamp.LAMP_ERR_UNSUPPORTED, "at most"),
    (dict(W=FAKE + 8), lamp.LAMP_ERR_UNSUPPORTED, "16-byte"),
    (dict(out=FAKE + 1), lamp.LAMP_ERR_UNSUPPORTED, "aligned"),
    (dict(n_selected_out=FAKE + 4), lamp.LAMP_ERR_UNSUPPORTED, "aligned"),
])
def test_gelu_argument_checks(lib, kw, code, msg):
    assert call_gelu(**kw) == code
    assert msg in lamp.lamp_last_error()


def test_gelu_null_args(lib):
    assert _native.load().lamp_linear_gelu(None) == lamp.LAMP_ERR_ARG


def call_ln(**kw):
    base = dict(M=4, N=40, K=16, x=FAKE, W=FAKE, out=FAKE, mu=4, tau=1.0)
    base.update(kw)
    return lamp.lamp_linear_layernorm(check=False, **base)


@pytest.mark.parametrize("kw,code,msg", [
    (dict(W=None), lamp.LAMP_ERR_ARG, "non-NULL"),
    (dict(N=0), lamp.LAMP_ERR_ARG, "positive"),
    (dict(mu=0), lamp.LAMP_ERR_ARG, "mu"),
    (dict(variant=lamp.LAMP_RELAXED), lamp.LAMP_ERR_ARG, "relaxed"),
    (dict(tau=float("nan")), lamp.LAMP_ERR_ARG, "tau"),
    (dict(variant=lamp.LAMP_GIVEN_MASK), lamp.LAMP_ERR_ARG, "mask_in"),
    (dict(eps=-1.0), lamp.LAMP_ERR_ARG, "eps"),
    (dict(scale=float("nan")), lamp.LAMP_ERR_ARG, "scale"),
    (dict(K=20), lamp.LAMP_ERR_UNSUPPORTED, "multiple of 8"),
    (dict(N=8193), lamp.LAMP_ERR_UNSUPPORTED, "at most 8192"),
    (dict(x=FAKE + 2), lamp.LAMP_ERR_UNSUPPORTED, "16-byte"),
    (dict(workspace=FAKE + 2), lamp.LAMP_ERR_UNSUPPORTED, "aligned"),
    (dict(workspace=FAKE, workspace_bytes=4 * 40 * 4 - 1), lamp.LAMP_ERR_WORKSPACE, "smaller"),
])
def test_ln_argument_checks(lib, kw, code, msg):
    assert call_ln(**kw) == code
    assert msg in lamp.lamp_last_error()


def test_ln_workspace_size(lib):
    assert lamp.lamp_ln_workspace_size(1024, 1600) == 1024 * 1600 * 4
    assert lamp.lamp_ln_workspace_size(0, 5) == 0


def test_plain_c_client_compiles_links_and_runs(lib, tmp_path):
    """A C program that includes only include/lamp.h links against liblamp.so and
    gets the documented errors back without a GPU."""
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.dirname(_native.LIB_PATH)
    exe = str(tmp_path / "abi_client")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(root, "include"),
                    os.path.join(root, "tests", "c_abi", "abi_client.c"), "-L", pkg, "-llamp",
                    f"-Wl,-rpath,{pkg}", "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert "abi client ok" in r.stdout
