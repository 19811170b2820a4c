"""The C-ABI library loads and exports every entry point include/orthrus.h
declares; host-only size queries and argument checks work without a GPU."""
import ctypes as C
import os
import re

import pytest

import synth
from shared_kv_draft_b200 import orthrus
from shared_kv_draft_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return orthrus.load()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "orthrus.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(orthrus_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 17
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(n for n, _, _ in orthrus.SIGNATURES) == names


def test_core_calls_declared():
    names = declared_symbols()
    for n in ("orthrus_draft_block", "orthrus_verify_block", "orthrus_accept_commit", "orthrus_decode_step"):
        assert n in names


def test_block_scratch_is_four_and_a_half_mib(lib):
    cfg = orthrus.make_config(synth.QWEN3_8B)
    assert orthrus.block_scratch_bytes(cfg, 1, 32) == 4_718_592


def test_size_queries_reject_bad_shapes(lib):
    cfg = orthrus.make_config(synth.QWEN3_8B)
    assert orthrus.plan_bytes(cfg) > 0
    assert orthrus.workspace_bytes(cfg, 1, 2048, 32, 33) > 0
    assert orthrus.workspace_bytes(cfg, 1, 2048, 65, 66 * 1) == 0      # K > 64
    assert orthrus.workspace_bytes(cfg, 2, 2048, 32, 33) == 0          # rows < batch*(K+1)
    bad = orthrus.make_config(synth.QWEN3_8B)
    bad.head_dim = 96
    assert orthrus.plan_bytes(bad) == 0
    bad = orthrus.make_config(synth.QWEN3_8B)
    bad.vocab = 1000
    assert orthrus.plan_bytes(bad) == 0
    off = orthrus.block_scratch_offset(cfg, 1, 2048, 32, 33)
    assert 0 < off < orthrus.workspace_bytes(cfg, 1, 2048, 32, 33)


def test_null_plan_is_rejected(lib):
    assert lib.orthrus_decode_step(None, None, 32, None, None, None, None) == orthrus.ERR_ARG
    assert lib.orthrus_draft_block(None, None, 4, None, None, None) == orthrus.ERR_ARG
    assert lib.orthrus_decode_step_launches(None, 4) == 0
    buf = C.create_string_buffer(64)  # not an initialised plan
    assert lib.orthrus_verify_block(buf, None, None, 4, None, None, None) == orthrus.ERR_ARG
    assert lib.orthrus_status_ptr(buf) is None


def test_plan_init_rejects_nulls(lib):
    cfg = orthrus.make_config(synth.TINY)
    n = orthrus.plan_bytes(cfg)
    buf = C.create_string_buffer(n)
    w = orthrus.Weights()
    cache = orthrus.Cache(None, None, None, 1, 64)
    code = lib.orthrus_plan_init(buf, n, C.byref(cfg), C.byref(w), C.byref(cache), 4, 5, None, 0, None)
    assert code == orthrus.ERR_ARG


def test_refine_and_sampling_calls_check_arguments_on_the_host(lib):
    nan, inf = float("nan"), float("inf")
    assert lib.orthrus_draft_refine(None, None, None, 4, None, None, None) == orthrus.ERR_ARG
    assert lib.orthrus_decode_step_ex(None, None, 4, 2, None, None, None, None) == orthrus.ERR_ARG
    assert lib.orthrus_accept_sample(None, None, None, None, None, 4, 1.0, None, None, None, None,
                                     None) == orthrus.ERR_ARG
    assert lib.orthrus_decode_step_sampled(None, None, 4, 1.0, None, None, None, None, None, None, None,
                                           None) == orthrus.ERR_ARG
    # temperature must be positive and finite; 1 <= vocab <= 262144; rows >= 0
    for t in (0.0, -1.0, nan, inf):
        assert lib.orthrus_sample_tokens(None, 1, 1024, t, None, None, None, None) == orthrus.ERR_ARG
    assert lib.orthrus_sample_tokens(None, 1, 0, 1.0, None, None, None, None) == orthrus.ERR_ARG
    assert lib.orthrus_sample_tokens(None, 1, 262145, 1.0, None, None, None, None) == orthrus.ERR_ARG
    assert lib.orthrus_sample_tokens(None, -1, 1024, 1.0, None, None, None, None) == orthrus.ERR_ARG
    assert lib.orthrus_sample_tokens(None, 1, 1024, 1.0, None, None, None, None) == orthrus.ERR_ARG  # NULL buffers
    assert lib.orthrus_sample_tokens(None, 0, 1024, 1.0, None, None, None, None) == orthrus.OK       # nothing to do


def test_header_is_plain_c():
    """include/orthrus.h is a C header: it compiles as C99 with no C++ or CUDA types."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    r = subprocess.run([gcc, "-std=c99", "-fsyntax-only", "-Wall", "-Wextra", "-Werror", "-x", "c",
                        os.path.join(ROOT, "include", "orthrus.h")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def declared_prototypes():
    """name -> list of parameter declarations, from include/orthrus.h."""
    text = open(os.path.join(ROOT, "include", "orthrus.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for m in re.finditer(r"\b(orthrus_[a-z_0-9]+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
        params = [p.strip() for p in m.group(2).replace("\n", " ").split(",")]
        out[m.group(1)] = [] if params == ["void"] else params
    return out


def ctype_of(param):
    """The ctypes type a parameter declaration must be bound with."""
    decl = re.sub(r"\s+", " ", param)
    if "*" in decl or decl.startswith("orthrus_stream"):
        return "pointer"
    base = decl.rsplit(" ", 1)[0].replace("const ", "")
    return {"int32_t": C.c_int32, "size_t": C.c_size_t, "float": C.c_float}[base]


def test_binding_signatures_match_the_header():
    protos = declared_prototypes()
    assert set(protos) == set(declared_symbols())
    for name, res, args in orthrus.SIGNATURES:
        params = protos[name]
        assert len(args) == len(params), (name, len(args), len(params))
        for a, p in zip(args, params):
            want = ctype_of(p)
            if want == "pointer":
                assert a is C.c_void_p or issubclass(a, C._Pointer), (name, p, a)
            else:
                assert a is want, (name, p, a)
