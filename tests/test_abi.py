"""The C ABI library builds for sm_100a, loads without a GPU, exports every
symbol include/swa.h declares, and rejects bad arguments on the host before
touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

import sliding_window_gqa_prefill_b200 as swa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    swa.build()
    return swa.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "swa.h")).read()
    return sorted(set(re.findall(r"^\s*(?:swa_status_t|size_t|const char \*|int)\s+(swa_\w+)\s*\(",
                                 text, re.M)))


def test_header_declares_the_four_operations():
    names = declared_symbols()
    for n in ("swa_prefill", "swa_prefill_chunk", "swa_cache_append", "swa_decode"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", swa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(swa_\w+)$", out, re.M))
    missing = [n for n in declared_symbols() if n not in exported]
    assert not missing, missing
    for n in declared_symbols():
        assert hasattr(lib, n)


def test_index_checked_library_exports_the_same_symbols():
    """libswa_debug.so (SWA_BOUNDS_CHECK) is the same ABI: it builds, loads
    without a GPU and exports every declared symbol."""
    swa.build(debug=True)
    out = subprocess.run(["nm", "-D", "--defined-only", swa.DEBUG_LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(swa_\w+)$", out, re.M))
    assert not [n for n in declared_symbols() if n not in exported]
    with swa.bounds_checked():
        L = swa.lib()
    assert L is not swa.lib() and L._name == swa.DEBUG_LIB_PATH
    assert L.swa_prefill(None, 0x1000, 0x1000, 0x1000, 1, 16, 4, 2, 128, 8, 0, 0.1, None) == \
        swa.SWA_ERR_INVALID_ARG


def test_null_and_bad_sizes_rejected_without_device(lib):
    null = None
    ok_ptr = 0x1000            # aligned, never dereferenced: checks fail first
    S = swa.SWA_ERR_INVALID_ARG
    assert lib.swa_prefill(null, ok_ptr, ok_ptr, ok_ptr, 1, 16, 4, 2, 128, 8, 0, 0.1, None) == S
    assert lib.swa_prefill(ok_ptr, ok_ptr, ok_ptr, ok_ptr + 2, 1, 16, 4, 2, 128, 8, 0, 0.1, None) == S
    assert lib.swa_prefill(ok_ptr, ok_ptr, ok_ptr, ok_ptr, 0, 16, 4, 2, 128, 8, 0, 0.1, None) == S
    assert lib.swa_prefill(ok_ptr, ok_ptr, ok_ptr, ok_ptr, 1, 16, 4, 2, 128, 0, 0, 0.1, None) == S
    assert lib.swa_prefill(ok_ptr, ok_ptr, ok_ptr, ok_ptr, 1, 16, 4, 2, 128, 8, 7, 0.1, None) == S
    assert lib.swa_prefill(ok_ptr, ok_ptr, ok_ptr, ok_ptr, 1, 16, 4, 2, 128, 8, 0, -1.0, None) == S
    assert lib.swa_prefill(ok_ptr, ok_ptr, ok_ptr, ok_ptr, 1, 16, 3, 2, 128, 8, 0, 0.1, None) == S
    assert lib.swa_prefill(ok_ptr, ok_ptr, ok_ptr, ok_ptr, 1, 16, 4, 2, 80, 8, 0, 0.1, None) == \
        swa.SWA_ERR_UNSUPPORTED
    # chunk longer than the window
    assert lib.swa_prefill_chunk(ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr,
                                 1, 65, 4, 2, 128, 64, 0.1, None) == S
    # append: T > W, null pos
    assert lib.swa_cache_append(ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, 1, 65, 2, 128, 64, None) == S
    assert lib.swa_cache_append(ok_ptr, ok_ptr, ok_ptr, ok_ptr, null, 1, 1, 2, 128, 64, None) == S
    # chunked prefill with sinks: negative S, null sink buffer with S > 0
    assert lib.swa_prefill_chunk_sinks(ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr,
                                       1, 128, 8, 2, 128, 256, -1, 0.1, None) == S
    assert lib.swa_prefill_chunk_sinks(ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, null, ok_ptr, ok_ptr, ok_ptr,
                                       1, 128, 8, 2, 128, 256, 4, 0.1, None) == S
    # decode: workspace too small
    assert lib.swa_decode(ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, 2, 8, 2, 128, 4096, 0.1,
                          ok_ptr, 16, None) == S


def test_workspace_size_and_status_strings(lib):
    assert lib.swa_decode_workspace_size(0, 32, 8, 128, 4096) == 0
    n = lib.swa_decode_workspace_size(64, 32, 8, 128, 4096)
    # (B*Hq*splits) rows of D floats, then one (m, l) pair per row; the
    # 4096-key window takes 4 splits of 1024 keys
    rows = 64 * 32 * 4
    assert n == ((rows * 128 * 4 + 255) // 256) * 256 + rows * 8
    assert lib.swa_status_string(0) == b"SWA_OK"
    assert lib.swa_status_string(4) == b"SWA_ERR_TIMEOUT"


def _ws(B, Hq, Hkv, D, splits):
    rows = B * Hq * splits
    return ((rows * D * 4 + 255) // 256) * 256 + rows * 8


@pytest.mark.parametrize("B,Hq,Hkv,W,splits", [
    (64, 32, 8, 4096, 4),      # full batch: splits of 1024 keys
    (8, 32, 8, 4096, 4),       # 8 x 8 x 4 = 256 blocks already
    (4, 32, 8, 4096, 8),       # small batches: shorter splits to reach ~256 blocks
    (2, 32, 8, 4096, 16),
    (1, 32, 8, 4096, 16),      # at least 256 keys per split
    (1, 32, 8, 100, 1),        # a window shorter than one split
    (3, 8, 2, 20000, 40),      # 512-key splits
    (1, 32, 2, 4096, 16),      # group of 16: two groups of 8 per K/V head, 4 groups in all
    (2, 22, 2, 4096, 6),       # group of 11 (prime): 11 groups of one head per K/V head (704-key splits)
])
def test_decode_split_policy_through_the_workspace_size(lib, B, Hq, Hkv, W, splits):
    """The split length (1024 keys, shorter down to 256 when B times the
    groups of the grid give under ~256 blocks) and the grouping of more than 8
    heads per K/V head both show in the workspace size, a host-only call."""
    assert lib.swa_decode_workspace_size(B, Hq, Hkv, 128, W) == _ws(B, Hq, Hkv, 128, splits)


def test_every_declared_operation_has_a_python_binding():
    """Each symbol of include/swa.h is reachable from Python: a wrapper of the
    same name, the rope_theta argument of the base wrapper for the *_rope
    entry points, or the error path (status string, last CUDA error)."""
    import inspect
    src = inspect.getsource(swa)
    for name in declared_symbols():
        if hasattr(swa, name):
            continue
        if name.endswith("_rope") and hasattr(swa, name[:-5]):
            assert "rope_theta" in inspect.signature(getattr(swa, name[:-5])).parameters, name
            assert f"lib().{name}(" in src, name
            continue
        assert name in ("swa_status_string", "swa_last_cuda_error"), name
        assert f".{name}(" in src, name
    for name in swa.__all__:
        assert hasattr(swa, name), name


def test_noalloc_binding_checks_its_arguments_on_the_host():
    import torch
    q = torch.zeros(2, 8, 128, dtype=torch.bfloat16)
    kc = torch.zeros(2, 64, 2, 128, dtype=torch.bfloat16)
    pos = torch.zeros(2, dtype=torch.int32)
    with pytest.raises(TypeError):
        swa.swa_decode_noalloc(q, kc, kc, pos, 0.1, out=torch.empty_like(q))


def test_product_path_does_not_use_the_oracle():
    """The package and its C sources never import, load or link the oracle;
    bench.py reaches it only in the CPU-baseline sampler that its cpu_baseline
    leg and its reference arm call."""
    import ast
    pkg = os.path.join(ROOT, "sliding_window_gqa_prefill_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "import oracle" not in text and "libswa_oracle" not in text, f
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    users = set()
    for fn in ast.walk(tree):
        if isinstance(fn, ast.FunctionDef):
            for node in ast.walk(fn):
                if isinstance(node, ast.Import) and any(a.name == "oracle" for a in node.names):
                    users.add(fn.name)
    top_level = [n for n in tree.body if isinstance(n, (ast.Import, ast.ImportFrom))
                 and any(a.name == "oracle" for a in n.names)]
    assert not top_level and users == {"cpu_oracle_sample"}, users
