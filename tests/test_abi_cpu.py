"""Host-side checks of the C ABI (no GPU): the library loads, exports every
function include/fvattn.h declares, and its size helpers and argument checks
behave as documented."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from top_routed_block_b200 import _build
    _build.build()
    import top_routed_block_b200 as fv
    return fv.load_library()


def declared_functions():
    with open(os.path.join(ROOT, "include", "fvattn.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fvattn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("fvattn_route", "fvattn_sparse_fwd", "fvattn_lpt_order", "fvattn_route_workspace_bytes",
                     "fvattn_fwd_workspace_bytes", "fvattn_route_max_nnz", "fvattn_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)


def test_only_declared_symbols_are_exported(lib):
    import subprocess
    from top_routed_block_b200 import LIB_PATH
    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l and l.split()[-1].startswith("fvattn_")}
    assert exported == set(declared_functions())


def test_header_is_plain_c(lib, tmp_path):
    """The boundary is a C ABI: the header compiles as strict C99 (and as C++), and
    a C program that calls a host-only entry point links against the library."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use.c"
    src.write_text('#include "fvattn.h"\n'
                   'int main(void) { return fvattn_attn_num_items(1, 40, 32760, 64) == 40 * 256 ? 0 : 1; }\n')
    inc = os.path.join(ROOT, "include")
    for cmd in (["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", inc, "-c", str(src),
                 "-o", str(tmp_path / "c.o")],
                ["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-I", inc, "-x", "c++", "-c", str(src),
                 "-o", str(tmp_path / "cpp.o")]):
        r = subprocess.run(cmd, capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
    from top_routed_block_b200 import LIB_PATH
    libdir = os.path.dirname(LIB_PATH)
    exe = tmp_path / "use"
    r = subprocess.run(["gcc", str(tmp_path / "c.o"), "-o", str(exe), "-L", libdir, "-lfvattn",
                        "-Wl,-rpath," + libdir], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert subprocess.run([str(exe)]).returncode == 0


def test_status_strings(lib):
    import top_routed_block_b200 as fv
    assert fv.status_string(0) == "ok"
    for code in range(-7, 0):
        assert fv.status_string(code) not in ("", "unknown status")
    assert fv.status_string(-99) == "unknown status"
    assert b"sm_100a" in lib.fvattn_build_info()


def test_size_helpers(lib):
    import top_routed_block_b200 as fv
    assert fv.fvattn_num_rows(1, 40, 32760, 128) == 40 * 256
    assert fv.fvattn_route_max_nnz(1, 24, 118800, 128) == 24 * 929 * 929
    assert fv.fvattn_route_max_nnz(0, 1, 1, 64) == 0
    rw = fv.fvattn_route_workspace_bytes(1, 40, 32760, 128, 128)
    # two fp64 block-mean tensors dominate: 2 * 40 * 256 * 128 * 8 bytes
    assert rw >= 2 * 40 * 256 * 128 * 8
    assert fv.fvattn_route_workspace_bytes(1, 1, 100, 96, 128) == 0      # d unsupported
    assert fv.fvattn_route_workspace_bytes(1, 1, 100, 64, 32) == 0       # block unsupported
    fw = fv.fvattn_fwd_workspace_bytes(1, 40, 32760, 128)
    # the work order: one int32 per CSR row, plus one rank per head
    assert fw >= 40 * 256 * 4 + 40 * 4
    assert fv.fvattn_fwd_workspace_bytes(1, 4097, 128, 128) == 0           # head limit 4096
    assert fv.fvattn_lpt_workspace_bytes(10, 5000) == 0                  # count limit 4096
    # work items: query blocks at block 128, pairs of query blocks (2i, 2i+1) at block 64
    assert fv.fvattn_attn_num_items(1, 40, 32760, 128) == 40 * 256
    assert fv.fvattn_attn_num_items(1, 40, 32760, 64) == 40 * 256          # 512 blocks per head, 256 pairs
    assert fv.fvattn_attn_num_items(2, 3, 900, 64) == 6 * 8                # 15 blocks: 7 pairs and one alone
    assert fv.fvattn_attn_num_items(1, 1, 50, 64) == 1
    assert fv.fvattn_attn_num_items(1, 1, 100, 32) == 0                    # block unsupported
    # block 64 also keeps the pairs' union sizes, their scan and per-head sums
    f64 = fv.fvattn_fwd_workspace_bytes(1, 40, 32760, 64)
    assert f64 >= 40 * 256 * 4 * 3 + 40 * 4 * 2


def test_invalid_arguments_rejected_before_any_device_work(lib):
    P = ctypes.c_void_p
    fake = P(16)  # never dereferenced: argument checks fail first
    # p outside (0, 1]
    for p in (0.0, -0.5, 1.5, float("nan")):
        rc = lib.fvattn_route(fake, fake, 1, 1, 128, 64, 64, p, fake, fake, 4, fake, fake, 1 << 20, fake, None)
        assert rc == -1
    # unsupported head dim / block
    assert lib.fvattn_route(fake, fake, 1, 1, 128, 96, 64, 0.5, fake, fake, 4, fake, fake, 1 << 20, fake, None) == -2
    assert lib.fvattn_sparse_fwd(fake, fake, fake, fake, fake, 1, 1, 128, 64, 32, 0, fake, fake, fake, 1 << 20,
                                 fake, None) == -2
    # null pointers
    assert lib.fvattn_sparse_fwd(None, fake, fake, fake, fake, 1, 1, 128, 64, 64, 0, fake, fake, fake, 1 << 20,
                                 fake, None) == -1
    # misaligned tensor pointer
    assert lib.fvattn_sparse_fwd(P(18), fake, fake, fake, fake, 1, 1, 128, 64, 64, 0, fake, fake, fake, 1 << 20,
                                 fake, None) == -3
    # workspace too small
    assert lib.fvattn_sparse_fwd(fake, fake, fake, fake, fake, 1, 1, 128, 64, 64, 0, fake, fake, fake, 8,
                                 fake, None) == -4
    # causal must be 0 or 1
    assert lib.fvattn_sparse_fwd(fake, fake, fake, fake, fake, 1, 1, 128, 64, 64, 2, fake, fake, fake, 1 << 20,
                                 fake, None) == -1
    # e4m3 quantization: unsupported d, null pointers, misaligned input
    assert lib.fvattn_quant_e4m3(fake, 1, 1, 128, 96, 64, fake, fake, None) == -2
    assert lib.fvattn_quant_e4m3(None, 1, 1, 128, 64, 64, fake, fake, None) == -1
    assert lib.fvattn_quant_e4m3(fake, 1, 1, 128, 64, 64, fake, None, None) == -1
    assert lib.fvattn_quant_e4m3(P(18), 1, 1, 128, 64, 64, fake, fake, None) == -3
    assert lib.fvattn_quant_e4m3(fake, 0, 1, 128, 64, 64, fake, fake, None) == -1
    # at most 4096 query blocks per sequence and 4096 heads, refused before any device work
    for block in (64, 128):
        assert lib.fvattn_sparse_fwd(fake, fake, fake, fake, fake, 1, 1, 4097 * block, 64, block, 0, fake, fake,
                                     fake, 1 << 30, fake, None) == -2
    assert lib.fvattn_sparse_fwd(fake, fake, fake, fake, fake, 1, 4097, 128, 64, 64, 0, fake, fake, fake, 1 << 30,
                                 fake, None) == -2
    assert lib.fvattn_sparse_bwd(fake, fake, fake, fake, fake, fake, fake, fake, 1, 1, 4097 * 128, 64, 128, 0,
                                 fake, fake, fake, fake, 1 << 30, fake, None) == -2
    # the block-64 work order reads the column indices and writes a status word
    assert lib.fvattn_attn_work_order(fake, None, 1, 1, 256, 64, fake, fake, 1 << 20, fake, None) == -1
    assert lib.fvattn_attn_work_order(fake, fake, 1, 1, 256, 64, fake, fake, 1 << 20, None, None) == -1
    assert lib.fvattn_attn_work_order(fake, None, 1, 1, 256, 32, fake, fake, 1 << 20, None, None) == -2
    # routing supports at most 1024 blocks per sequence
    assert lib.fvattn_route(fake, fake, 1, 1, 1025 * 64, 64, 64, 0.5, fake, fake, 4, fake, fake, 1 << 30, fake,
                            None) == -2


def test_binding_fails_loudly_without_library(tmp_path):
    import top_routed_block_b200 as fv
    saved = fv._lib
    try:
        fv._lib = None
        with pytest.raises(fv.FvattnError):
            fv.load_library(str(tmp_path / "missing.so"))
    finally:
        fv._lib = saved


def test_noalloc_rejects_shapes_beyond_its_scratch_without_a_gpu(lib):
    # Null pointers everywhere: the size check must fail first; were it to regress,
    # the null-pointer check would still stop the call before any device work.
    B, H, N, block = 16, 256, 65536, 128
    assert lib.fvattn_sparse_fwd_noalloc(None, None, None, None, None, B, H, N, 128, block, 0, None, None, None,
                                         None) == -4


def test_rlb_plan_matches_the_oracle(lib, oracle_mod):
    # host-only entry point: the library's plan equals the oracle's on random instances
    import numpy as np
    import top_routed_block_b200 as fv
    rng = np.random.default_rng(11)
    for ranks, units in [(1, 3), (2, 4), (3, 7), (8, 5), (8, 40), (16, 3)]:
        for _ in range(5):
            work = (rng.integers(0, 300, size=(ranks, units)) * (rng.random((ranks, 1)) * 3)).astype(np.int64)
            want = oracle_mod.rlb_plan(work).tolist()
            assert [list(m) for m in fv.fvattn_rlb_plan(work)] == want
    assert fv.fvattn_rlb_plan(np.array([[3, 4], [4, 3]])) == []
    with pytest.raises(fv.FvattnError):
        fv.fvattn_rlb_plan(np.array([[1, -1]]))
    with pytest.raises(fv.FvattnError):
        fv.fvattn_rlb_plan(np.array([[4, 4, 4], [1, 1, 0], [1, 0, 0]]), max_moves=1)   # needs 3 moves
