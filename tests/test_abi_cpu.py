"""The C ABI without a GPU: the library loads, exports every symbol include/mla.h declares, and
rejects invalid requests on the host before any launch (no compute calls here)."""
import ctypes
import os
import re

import pytest

from head_latent_attention_08_b200 import build as B
from head_latent_attention_08_b200 import mla as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return M.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "mla.h")).read()
    return sorted(set(re.findall(r"^MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_binding_names():
    assert set(declared_symbols()) == set(M.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_abi_version_and_status_strings(lib):
    assert lib.mla_abi_version() == 3
    for s in range(10):
        assert lib.mla_status_string(s)
    assert b"unknown" in lib.mla_status_string(1234)


def _d(**kw):
    base = dict(n_heads=4, kv_lora_rank=16, rope_dim=8, qk_nope=8, v_head=8, d_model=32)
    base.update(kw)
    return M.dims(**base)


FAKE = 0x10000  # a non-NULL, 256-aligned address that validation must reject before use


def test_validation_errors_return_before_launch(lib):
    d = _d()
    # NULL dims, bad dtype, bad mode / flags
    assert lib.mla_absorb_weights(None, 0, 0, FAKE, FAKE, FAKE, 1, FAKE, None) == 1
    assert lib.mla_absorb_weights(ctypes.byref(d), 7, 0, FAKE, FAKE, FAKE, 1, FAKE, None) == 3
    assert lib.mla_absorb_weights(ctypes.byref(d), 0, 42, FAKE, FAKE, FAKE, 1, FAKE, None) == 9
    assert lib.mla_append_latent(ctypes.byref(d), 1, FAKE, 10, FAKE, FAKE, FAKE, FAKE, 1, 8, 1e-6, 1e4, None) == 9
    assert lib.mla_decode_absorbed(ctypes.byref(d), 1, FAKE, FAKE, FAKE, 1, 1, 4, 4, 4, FAKE, None,
                                   FAKE, 1 << 20, None) == 9
    assert lib.mla_linear(0, FAKE, FAKE, 2, 2, 2, 4, FAKE, None) == 9
    # NULL operands
    assert lib.mla_absorb_weights(ctypes.byref(d), 0, 0, None, FAKE, FAKE, 1, FAKE, None) == 1
    assert lib.mla_append_latent(ctypes.byref(d), 1, None, 10, FAKE, FAKE, FAKE, FAKE, 1, 0, 1e-6, 1e4, None) == 1
    assert lib.mla_decode_absorbed(ctypes.byref(d), 1, None, FAKE, FAKE, 1, 1, 4, 4, 0, FAKE, None,
                                   FAKE, 1 << 20, None) == 1
    assert lib.mla_out_project(ctypes.byref(d), 1, None, FAKE, FAKE, None, 2, FAKE, FAKE, 1 << 20, None) == 1
    # bad sizes
    bad = _d(n_heads=0)
    assert lib.mla_absorb_weights(ctypes.byref(bad), 0, 0, FAKE, FAKE, FAKE, 1, FAKE, None) == 2
    assert lib.mla_absorb_weights(ctypes.byref(d), 0, 0, FAKE, FAKE, FAKE, -1, FAKE, None) == 2
    odd = _d(rope_dim=7)
    assert lib.mla_append_latent(ctypes.byref(odd), 1, FAKE, 10, FAKE, FAKE, FAKE, FAKE, 1, 2, 1e-6, 1e4, None) == 2
    # sum of lengths larger than batch * max_seqlen
    assert lib.mla_decode_absorbed(ctypes.byref(d), 1, FAKE, FAKE, FAKE, 2, 1, 4, 9, 0, FAKE, None,
                                   FAKE, 1 << 20, None) == 2
    # causal with fewer positions than query tokens
    assert lib.mla_decode_absorbed(ctypes.byref(d), 1, FAKE, FAKE, FAKE, 1, 4, 2, 2, 1, FAKE, None,
                                   FAKE, 1 << 20, None) == 2
    # misaligned bf16 operands and workspace
    assert lib.mla_absorb_weights(ctypes.byref(d), 1, 0, FAKE + 2, FAKE, FAKE, 1, FAKE, None) == 4
    assert lib.mla_decode_absorbed(ctypes.byref(d), 1, FAKE, FAKE, FAKE, 1, 1, 4, 4, 0, FAKE, None,
                                   FAKE + 16, 1 << 20, None) == 4
    # workspace too small for the projection
    assert lib.mla_out_project(ctypes.byref(d), 1, FAKE, FAKE, FAKE, None, 2, FAKE, FAKE, 16, None) == 5
    # empty problems are no-ops
    assert lib.mla_linear(0, None, None, 0, 5, 5, 0, None, None) == 0
    assert lib.mla_decode_absorbed(ctypes.byref(d), 1, None, None, None, 0, 1, 0, 0, 0, None, None,
                                   None, 0, None) == 0


def test_workspace_size_queries(lib):
    d = _d()
    n = ctypes.c_size_t(0)
    assert lib.mla_out_project_workspace_size(ctypes.byref(d), 1, 3, ctypes.byref(n)) == 0
    assert n.value >= 3 * 4 * 8 * 2
    assert lib.mla_decode_workspace_size(ctypes.byref(d), 0, 2, 1, 64, 100, 0, ctypes.byref(n)) == 0
    assert lib.mla_decode_workspace_size(ctypes.byref(d), 0, 2, 1, 64, 100, 0, None) == 1
    assert lib.mla_set_wait_limit(-1) == 2
    assert lib.mla_set_wait_limit(0) == 0


def test_binding_raises_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(M, "_lib", None)
    monkeypatch.setattr(M, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        M.lib()


def test_library_sources_allocate_no_device_memory():
    """The library allocates nothing: no CUDA allocation or free call and no torch allocator anywhere in
    its sources (the no-alloc decode and the workspace decode share every kernel and host helper).
    Comments are ignored; a pair of allocate and free calls inside a call would not show in a
    free-memory check, so this scan is the primary check."""
    import glob
    import re
    csrc = os.path.join(ROOT, "head_latent_attention_08_b200", "csrc")
    banned = re.compile(r"\b(cudaMalloc\w*|cudaFree\w*|cuMemAlloc\w*|cuMemFree\w*|cudaHostAlloc|"
                        r"cudaMallocHost|malloc|calloc|realloc|torch|c10|at::)\b")
    hits = []
    for path in sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh"))):
        code = re.sub(r"/\*.*?\*/", "", open(path, encoding="utf-8").read(), flags=re.S)
        for n, line in enumerate(code.splitlines(), 1):
            line = re.sub(r"//.*$", "", line)
            if banned.search(line):
                hits.append(f"{os.path.basename(path)}:{n}: {line.strip()}")
    assert not hits, "\n".join(hits)
