"""The C-ABI library loads and exports every symbol include/hs2.h declares;
host-side argument checks answer without a GPU (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "hs2.h")).read()
    return sorted(set(re.findall(r"HS2_API\s+[\w\s\*]+?\b(hs2_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def hs2():
    import token_level_kv_b200 as m
    return m


def test_header_declares_the_four_path_calls():
    names = _declared()
    for n in ("hs2_bridge_kv", "hs2_full_attn_select", "hs2_sparse_attn_prefill", "hs2_sparse_attn_decode"):
        assert n in names


def test_every_declared_symbol_is_exported(hs2):
    lib = ctypes.CDLL(hs2.LIB_PATH)
    for n in _declared():
        assert hasattr(lib, n), n
    assert set(_declared()) == set(hs2.EXPORTS)


def test_status_strings_and_version(hs2):
    assert hs2.lib.hs2_status_string(0) == b"HS2_OK"
    assert hs2.lib.hs2_status_string(5) == b"HS2_ERR_TIMEOUT"
    assert hs2.hs2_version().startswith("hs2")


def test_argument_checks_need_no_device(hs2):
    lib = hs2.lib
    assert lib.hs2_bridge_kv(None, 10, 2048, None, None, 256, 0, None, None, None, None, None) == 1
    assert b"null" in lib.hs2_last_error()
    # a misaligned pointer is refused before any CUDA call
    assert lib.hs2_bridge_kv(8, 10, 2048, 16, 16, 256, 0, 16, 16, None, None, None) == 1
    assert b"aligned" in lib.hs2_last_error()
    assert lib.hs2_bridge_kv(16, 10, 2048, 16, 16, 128, 0, 16, 16, None, None, None) == 2
    assert lib.hs2_sparse_attn_prefill(16, 16, 16, 16, 4, 100, 1152, 12, 256, 0.0625, 16, None) == 2
    assert lib.hs2_full_attn_select(16, 16, 16, None, None, 0, 1, 0, 4, 100, 100, 16, 256, 128, 1024,
                                    0.0625, 16, 16, None, 0, None) == 3


def test_workspace_sizes(hs2):
    n = ctypes.c_size_t(0)
    assert hs2.lib.hs2_full_attn_select_workspace(0, 1, 32768, 32768, 16, 256, 128, 1024, ctypes.byref(n)) == 0
    assert n.value >= 32768 * 32768 * 4 + 32768 * 16 * 8          # scores + (m, l)
    assert hs2.lib.hs2_full_attn_select_workspace(1, 64, 1, 131072, 16, 256, 128, 1024, ctypes.byref(n)) == 0
    assert n.value >= 64 * 16 * 131072 * 4                         # staged logits
    assert hs2.lib.hs2_full_attn_select_workspace(0, 1, 1, 10, 12, 256, 128, 1024, ctypes.byref(n)) == 2


def test_cpu_tensors_are_refused_by_the_binding(hs2):
    import torch
    x = torch.zeros(4, 16, 256, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        hs2.hs2_sparse_attn_prefill(x, x[0], x[0], torch.zeros(4, 8, dtype=torch.int32), x)


def test_header_compiles_as_c_and_cpp(tmp_path):
    import shutil
    import subprocess
    src = tmp_path / "use_hs2.c"
    src.write_text('#include "hs2.h"\nint main(void) { return (int)HS2_OK; }\n')
    for cc, std in (("gcc", "-std=c99"), ("g++", "-std=c++17")):
        if shutil.which(cc) is None:
            pytest.skip(f"{cc} not available")
        lang = ["-x", "c++"] if cc == "g++" else []
        r = subprocess.run([cc, std, "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), *lang,
                            "-c", str(src), "-o", str(tmp_path / f"use_{cc}.o")], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_shard_call_argument_checks_need_no_device(hs2):
    lib = hs2.lib
    n = ctypes.c_size_t(0)
    # bad sizes and shapes are refused before any CUDA call
    assert lib.hs2_decode_shard_workspace(0, 1000, 1152, 16, 256, 1024, ctypes.byref(n)) == 1
    assert lib.hs2_decode_shard_workspace(4, 1000, 1152, 12, 256, 1024, ctypes.byref(n)) == 2
    assert lib.hs2_decode_shard_attn(None, 16, 16, 16, 16, 4, 1000, 1000, 16, 256, 1024, 0.0625, 16, 16,
                                     16, 1 << 20, None) == 1
    assert lib.hs2_partial_merge(None, 2, 0, 16, 16, 4, 16, 256, None) == 1
    assert lib.hs2_partial_merge(16, 2, 2, 16, 16, 4, 16, 256, None) == 1            # shard >= n_shards
    assert lib.hs2_partial_finalize(16, 16, 16, 4, 12, 256, None) == 2               # Hq must be 8 or 16
    assert lib.hs2_decode_merge_candidates(None, 2, 4, 10000, 128, 1024, 16, None) == 1
    assert lib.hs2_decode_merge_candidates(16, 65, 4, 10000, 128, 1024, 16, None) == 2   # at most 64 shards
    assert b"64" in lib.hs2_last_error()
    assert lib.hs2_decode_shard_candidates(16, 1 << 20, 70000, 1000, 0, 1000, 16, 256, 128, 1024, 16, 16,
                                           None) == 1                                    # batch > 65535
    assert lib.hs2_sparse_decode_shard(16, 16, 16, 16, 16, 4, 1000, 1000, -1, 16, 1152, 16, 256, 0.0625, 16, 16,
                                       16, 1 << 20, None) != 0                           # negative shard offset
