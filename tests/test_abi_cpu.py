"""The C ABI library: it loads, exports what include/spa.h declares, and rejects
bad arguments on the host before touching a GPU.  No compute calls here."""
import ctypes
import os
import re
import shutil
import subprocess

import pytest
import torch

from head_partitioned_sparse_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spa.h")


@pytest.fixture(scope="module")
def lib():
    from head_partitioned_sparse_b200 import build
    build.build()
    return B.load()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^SPA_API\s+[\w\s\*]+?\b(spa_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("spa_create", "spa_destroy", "spa_index_append", "spa_select", "spa_decode",
                     "spa_workspace_size", "spa_last_error", "spa_device_status"):
        assert required in names
    assert sorted(B.EXPORTED) == names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (spa_\w+)", out))
    assert set(declared_functions()) <= exported
    # nothing but the C ABI is exported by name
    assert exported == set(declared_functions())


def declared_prototypes():
    """name -> (return type, [parameter types]) of every SPA_API function in the header."""
    text = re.sub(r"/\*.*?\*/", " ", open(HEADER).read(), flags=re.S)
    protos = {}
    for ret, name, params in re.findall(r"^SPA_API\s+([\w\s\*]+?)\b(spa_\w+)\s*\(([^;{]*?)\)\s*;", text, flags=re.M):
        params = " ".join(params.split())
        types = [] if params in ("", "void") else [p.strip().rsplit(" ", 1)[0] if not p.strip().endswith("*")
                                                  else p.strip() for p in params.split(",")]
        # a parameter "const float* x" keeps its type part: drop the name after the last '*'
        types = [re.sub(r"\s*\b\w+$", "", t) if "*" in t and not t.endswith("*") else t for t in types]
        protos[name] = (" ".join(ret.split()), types)
    return protos


def _ctype_kind(c_type: str) -> str:
    t = c_type.replace("const ", "").strip()
    if "*" in t or t in ("spa_handle", "spa_stream"):
        return "ptr"
    return {"int": "i32", "int64_t": "i64", "float": "f32", "double": "f64", "unsigned": "u32",
            "size_t": "size"}[t]


def _py_kind(ct) -> str:
    if ct in (ctypes.c_void_p, ctypes.c_char_p) or isinstance(ct, type) and issubclass(ct, ctypes._Pointer):
        return "ptr"
    return {ctypes.c_int: "i32", ctypes.c_int64: "i64", ctypes.c_float: "f32", ctypes.c_double: "f64",
            ctypes.c_uint: "u32", ctypes.c_size_t: "size"}[ct]


def test_binding_signatures_match_the_header_prototypes():
    """Every ctypes signature has the header's parameter count and, position by position,
    the same kind of argument (pointer, 32/64-bit integer, float, double, size)."""
    protos = declared_prototypes()
    assert sorted(protos) == sorted(B._SIGS)
    for name, (ret, params) in protos.items():
        py_ret, py_args = B._SIGS[name]
        assert len(py_args) == len(params), (name, params)
        assert [_py_kind(a) for a in py_args] == [_ctype_kind(t) for t in params], name
        assert _py_kind(py_ret) == ("i32" if ret == "spa_status" else _ctype_kind(ret)), name


def _cfg(**kw):
    base = dict(max_batch=2, n_q_heads=8, n_kv_heads=2, max_ctx=4096, kv_dtype=B.SPA_BF16,
                P_q=0x10000, P_k=0x20000)   # never dereferenced by the host checks
    base.update(kw)
    return B.make_config(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=64), B.SPA_ERR_UNSUPPORTED),
    (dict(idx_dim=8), B.SPA_ERR_UNSUPPORTED),
    (dict(kv_dtype=7), B.SPA_ERR_UNSUPPORTED),
    (dict(n_q_heads=6, n_kv_heads=2), B.SPA_ERR_UNSUPPORTED),     # G = 3
    (dict(n_q_heads=32, n_kv_heads=2), B.SPA_ERR_UNSUPPORTED),    # G = 16
    (dict(n_q_heads=7, n_kv_heads=2), B.SPA_ERR_INVALID_ARG),
    (dict(max_ctx=0), B.SPA_ERR_INVALID_ARG),
    (dict(max_ctx=(1 << 24) + 1), B.SPA_ERR_INVALID_ARG),
    (dict(max_batch=0), B.SPA_ERR_INVALID_ARG),
    (dict(split_rows=100), B.SPA_ERR_INVALID_ARG),
    (dict(P_q=None), B.SPA_ERR_INVALID_ARG),
    (dict(P_k=0x20004), B.SPA_ERR_INVALID_ARG),                    # misaligned
    (dict(rope_theta=-1.0), B.SPA_ERR_INVALID_ARG),
])
def test_config_validation(lib, kw, status):
    with pytest.raises(B.SpaError) as e:
        B.spa_workspace_size(_cfg(**kw))
    assert e.value.status == status
    assert B.spa_last_error()


def test_workspace_size_grows_with_context(lib):
    a = B.spa_workspace_size(_cfg(max_ctx=4096))
    b = B.spa_workspace_size(_cfg(max_ctx=8192))
    assert 0 < a < b
    # dominated by per-token buffers: probabilities, candidates, list (16 B/token/slice) + splits
    assert b - a >= 2 * 2 * 4096 * 16


def test_null_handle_is_rejected_without_a_device(lib):
    with pytest.raises(B.SpaError) as e:
        B.spa_decode(None, 16, 16, 16, 16, [1, 0], 16, 1, 0, 0.9, 4, 16, 16, None, stream=0)
    assert e.value.status == B.SPA_ERR_INVALID_ARG
    with pytest.raises(B.SpaError) as e:
        B.spa_index_append(None, 16, 16, 1, 1, 16, stream=0)
    assert e.value.status == B.SPA_ERR_INVALID_ARG
    with pytest.raises(B.SpaError) as e:
        B.spa_select(None, 16, 16, [1, 0], 16, 1, 0, 0.9, 4, 16, 16, 16, stream=0)
    assert e.value.status == B.SPA_ERR_INVALID_ARG
    assert B.spa_destroy(None) is None


def test_kernel_names(lib):
    names = [B.spa_kernel_name(i) for i in range(B.SPA_K_COUNT)]
    assert names[B.SPA_K_ATTEND] == "attend" and all(names)
    assert B.spa_kernel_name(99) == ""


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_create_without_device_fails_loudly(lib):
    with pytest.raises(B.SpaError) as e:
        B.spa_create(_cfg())
    assert e.value.status in (B.SPA_ERR_CUDA, B.SPA_ERR_UNSUPPORTED)


def test_context_parallel_calls_reject_a_null_handle(lib):
    for call in (lambda: B.spa_cp_exchange_sizes(None, 1, 2, [1, 0]),
                 lambda: B.spa_cp_combine(None, 16, 16, 2, 1, 16, stream=0),
                 lambda: B.spa_cp_phase(None, B.SPA_CP_STATS, B.make_cp_args(
                     q_pre=16, k_cache=16, v_cache=16, idx_cache=16, head_mask=[1, 0], seq_lens=16, B=1, p=0.9,
                     n_sink=4, window=16, n_ranks=2, rank=0, pos0=0, max_seq_len=0, stats=16, hist1=16, hist2=16,
                     hist3=16, out_all=16, lse_all=16), stream=0)):
        with pytest.raises(B.SpaError) as e:
            call()
        assert e.value.status == B.SPA_ERR_INVALID_ARG


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_cp_args_layout_matches_the_header(tmp_path):
    """The ctypes mirror of spa_cp_args has the C layout (size and every field offset)."""
    fields = [f for f, _ in B.spa_cp_args._fields_]
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "spa.h"\nint main(void) {\n'
                   '  printf("%zu", sizeof(spa_cp_args));\n'
                   + "".join(f'  printf(" %zu", offsetof(spa_cp_args, {f}));\n' for f in fields)
                   + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()]
    want = [ctypes.sizeof(B.spa_cp_args)] + [getattr(B.spa_cp_args, f).offset for f in fields]
    assert got == want
