"""CPU checks of the C ABI: the library loads, exports every declared symbol,
its host-only helper is right, and bad arguments are refused before any
device work.  No call here reaches the GPU."""

import ctypes as C
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tokengate.h")


@pytest.fixture(scope="module")
def lib():
    from learned_token_pruning_rmsnorm_b200 import build
    build.build()
    from learned_token_pruning_rmsnorm_b200 import _lib
    return _lib.load()


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(tg_[a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_five_stage_calls():
    names = _declared_functions()
    for n in ("tg_score", "tg_select_topk", "tg_compact", "tg_gated_attention", "tg_gated_prefill_layer"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from learned_token_pruning_rmsnorm_b200 import _lib
    names = _declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), f"{n} declared in tokengate.h but not exported"
        assert n in _lib.SIGNATURES, f"{n} has no binding signature"


_C_PROGRAM = r"""
#include "tokengate.h"
#include <stdio.h>
#include <string.h>

int main(void) {
    int32_t span[4] = {2, 8, 0, 15}, k[2] = {3, -1}, next[4];
    tg_status st;
    if (tg_abi_version() != 5) return 1;
    /* host-only helper: the next gate's span in this gate's kept order */
    if (tg_next_gate_span(span, k, 2, next) != TG_OK) return 2;
    if (next[0] != 2 || next[1] != 5 || next[2] != 0 || next[3] != 15) return 3;
    /* refused before any device work: D = 100 is not a multiple of 64 */
    st = tg_score(NULL, NULL, NULL, 1, 128, 100, NULL, NULL, NULL, 0.0f, 64, 1e-6f, NULL, NULL);
    if (st != TG_ERR_UNSUPPORTED) return 4;
    if (strstr(tg_last_error_string(), "D=100") == NULL) return 5;
    if (tg_gated_attention_backward_workspace_size(7, 3, 1, 64) != (size_t)(132 + 2688) * 4) return 6;
    printf("ok\n");
    return 0;
}
"""


def test_header_compiles_as_c_and_the_library_links(lib, tmp_path):
    """The header is plain C (C11, warnings as errors) and a C program links the
    library and calls it without PyTorch (host-side entry points only)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no gcc")
    pkg = os.path.join(ROOT, "learned_token_pruning_rmsnorm_b200")
    src = tmp_path / "prog.c"
    src.write_text(_C_PROGRAM)
    exe = tmp_path / "prog"
    cmd = [gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           str(src), "-L", pkg, "-ltokengate", "-Wl,-rpath," + pkg, "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)


def test_abi_version(lib):
    assert lib.tg_abi_version() == 5


def test_kept_count_host_helper(lib):
    from learned_token_pruning_rmsnorm_b200 import tg_kept_count
    tot, cu_kept = tg_kept_count([0, 10, 10, 25, 40], [[2, 8], [0, 0], [0, 15], [5, 5]], [3, 4, -1, 0])
    assert tot == 37 and cu_kept.tolist() == [0, 7, 7, 22, 37]
    # against the workload shape helper for every configured workload
    from workloads import CONFIGS
    for w in CONFIGS.values():
        tot, cu_kept = tg_kept_count(w.cu_seqlens(), w.span_array(), w.budget_array())
        np.testing.assert_array_equal(cu_kept, w.cu_kept())


def test_kept_count_rejects_bad_spans(lib):
    from learned_token_pruning_rmsnorm_b200 import TokenGateError, tg_kept_count
    with pytest.raises(TokenGateError):
        tg_kept_count([0, 10], [[5, 11]], [1])
    with pytest.raises(TokenGateError):
        tg_kept_count([0, 10], [[6, 5]], [1])


def test_invalid_shapes_are_refused_before_launch(lib):
    from learned_token_pruning_rmsnorm_b200 import _lib
    P = C.c_void_p(16)  # never dereferenced: validation fails first
    # D not a multiple of 64
    st = lib.tg_score(P, P, P, 1, 128, 100, P, P, P, 0.0, 64, 1e-6, P, None)
    assert st == _lib.TG_ERR_UNSUPPORTED
    assert b"D=100" in lib.tg_last_error_string()
    # I above 256
    st = lib.tg_score(P, P, P, 1, 128, 256, P, P, P, 0.0, 512, 1e-6, P, None)
    assert st == _lib.TG_ERR_UNSUPPORTED
    # head_dim 96
    st = lib.tg_gated_attention(P, P, P, P, 1, 10, 10, 4, 2, 96, P, P, P, P, P, 0.1, P, None, None, 0, None)
    assert st == _lib.TG_ERR_UNSUPPORTED
    # head_dim 256 is supported (an empty batch returns before any device work) and
    # never needs the causal-split scratch (one query head per CTA)
    st = lib.tg_gated_attention(P, P, P, P, 0, 0, 0, 8, 2, 256, P, P, P, P, P, 0.1, P, None, None, 0, None)
    assert st == _lib.TG_OK
    assert lib.tg_gated_attention_workspace_size(1, 32768, 16, 8, 256) == 0
    # Hq not a multiple of Hkv
    st = lib.tg_gated_attention(P, P, P, P, 1, 10, 10, 6, 4, 64, P, P, P, P, P, 0.1, P, None, None, 0, None)
    assert st == _lib.TG_ERR_INVALID_ARG
    # null pointers
    st = lib.tg_select_topk(None, P, P, P, 1, 10, P, None, None, None, None, None, None)
    assert st == _lib.TG_ERR_INVALID_ARG
    st = lib.tg_select_topk(P, P, P, P, 1, 10, P, P, P, None, None, None, None)  # map without pos/rank/gls
    assert st == _lib.TG_ERR_INVALID_ARG
    st = lib.tg_compact(P, P, P, P, P, 1, 10, 64, P, 20, P, P, P, P, P, None)  # M > T
    assert st == _lib.TG_ERR_INVALID_ARG
    st = lib.tg_gated_prefill_layer(None, None)
    assert st == _lib.TG_ERR_INVALID_ARG


def test_backward_workspace_size_matches_its_documentation(lib):
    """6 floats per (row, head), each of the three sections padded to 16 bytes, plus fp32
    partial dk and dv per query head for GQA groups outside 1, 2, 4 and 8 (those reduce
    inside a thread-block cluster or need no reduction), and for every group of two or more
    at head_dim 256 (no cluster reduction there)."""
    def expect(M, Hq, Hkv, d):
        mh = M * Hq
        rows = 4 * mh + 2 * ((mh + 3) // 4 * 4)
        grp = Hq // Hkv
        parts = 2 * grp * M * Hkv * d if grp > 1 and (d == 256 or grp not in (2, 4, 8)) else 0
        return (rows + parts) * 4
    for M, Hq, Hkv, d in [(2256, 16, 8, 128), (7, 3, 1, 64), (10, 8, 1, 64), (5, 4, 4, 128), (9, 6, 1, 128),
                          (1, 8, 2, 64), (33, 12, 1, 64), (2384, 8, 2, 256), (7, 3, 3, 256), (9, 6, 1, 256)]:
        assert lib.tg_gated_attention_backward_workspace_size(M, Hq, Hkv, d) == expect(M, Hq, Hkv, d), (M, Hq, Hkv, d)


def test_prefill_workspace_size_matches_its_documentation(lib):
    """tg_gated_prefill_workspace_size: the attention's scratch rounded up to 256 bytes, then
    the selection's [B][2048] int32 first-pass histogram; the histogram alone without
    attention layers; 0 for an empty batch."""
    for B, max_M, Hq, Hkv, d in [(1, 2256, 16, 8, 128), (4, 65536, 16, 8, 128), (1, 2384, 8, 2, 256),
                                 (3, 700, 6, 3, 64), (2, 100, 8, 8, 128)]:
        attn = lib.tg_gated_attention_workspace_size(B, max_M, Hq, Hkv, d)
        want = (attn + 255) // 256 * 256 + B * 2048 * 4
        assert lib.tg_gated_prefill_workspace_size(B, max_M, Hq, Hkv, d, 1) == want, (B, max_M, Hq, Hkv, d)
        assert lib.tg_gated_prefill_workspace_size(B, max_M, Hq, Hkv, d, 0) == B * 2048 * 4
    assert lib.tg_gated_prefill_workspace_size(0, 100, 8, 8, 128, 1) == 0


def test_attention_workspace_covers_both_kernels(lib, monkeypatch):
    """The workspace size does not depend on which two-head kernel runs
    (TG_ATTENTION_KERNEL): it is the larger of the two kernels' causal-split needs."""
    sizes = {}
    for choice in (None, "persistent", "per_unit"):
        if choice is None:
            monkeypatch.delenv("TG_ATTENTION_KERNEL", raising=False)
        else:
            monkeypatch.setenv("TG_ATTENTION_KERNEL", choice)
        sizes[choice] = [lib.tg_gated_attention_workspace_size(B, M, 16, 8, 128)
                         for B, M in [(1, 2256), (1, 16384), (2, 9000), (4, 40000)]]
    assert sizes[None] == sizes["persistent"] == sizes["per_unit"]
    assert all(n > 0 for n in sizes[None][:1])


def test_empty_batches_are_no_ops(lib):
    from learned_token_pruning_rmsnorm_b200 import _lib
    assert lib.tg_select_topk(None, None, None, None, 0, 0, None, None, None, None, None, None, None) == _lib.TG_OK
    assert lib.tg_score(None, None, None, 0, 0, 64, None, None, None, 0.0, 16, 1e-6, None, None) == _lib.TG_OK


def test_missing_library_fails_loudly(monkeypatch):
    from learned_token_pruning_rmsnorm_b200 import _lib
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", os.path.join(ROOT, "no_such_dir", "libtokengate.so"))
    with pytest.raises(ImportError):
        _lib.load()


def test_product_code_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "learned_token_pruning_rmsnorm_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "tg_oracle" not in src and "liboracle" not in src, f


def test_gather_rows_refuses_bad_rows_before_launch(lib):
    from learned_token_pruning_rmsnorm_b200 import _lib
    P = C.c_void_p(16)  # never dereferenced: validation fails first
    st = lib.tg_gather_rows(P, 10, 24, P, 4, P, None)  # 24-byte rows: not a multiple of 16
    assert st == _lib.TG_ERR_UNSUPPORTED
    assert b"row_bytes=24" in lib.tg_last_error_string()
    st = lib.tg_gather_rows(C.c_void_p(8), 10, 32, P, 4, P, None)  # misaligned source
    assert st == _lib.TG_ERR_INVALID_ARG
    assert lib.tg_gather_rows(None, 0, 32, None, 0, None, None) == _lib.TG_OK  # nothing to gather


def test_gather_rows_refuses_overlapping_buffers(lib):
    """The gather reads src and writes dst through restrict pointers (all of a row's loads
    before its stores), so in-place and overlapping calls are refused before any launch."""
    from learned_token_pruning_rmsnorm_b200 import _lib
    P = C.c_void_p(1 << 20)  # never dereferenced: validation fails first
    st = lib.tg_gather_rows(P, 100, 64, C.c_void_p(16), 10, P, None)  # src == dst
    assert st == _lib.TG_ERR_INVALID_ARG
    assert b"overlap" in lib.tg_last_error_string()
    # dst starts inside src's 100 rows of 64 bytes; src starts inside dst's 10 rows
    assert lib.tg_gather_rows(P, 100, 64, C.c_void_p(16), 10, C.c_void_p((1 << 20) + 99 * 64), None) == \
        _lib.TG_ERR_INVALID_ARG
    assert lib.tg_gather_rows(C.c_void_p((1 << 20) + 9 * 64), 100, 64, C.c_void_p(16), 10, P, None) == \
        _lib.TG_ERR_INVALID_ARG


def test_library_exports_only_the_c_abi(lib):
    """Only the tg_* entry points of tokengate.h are dynamic symbols: the launchers, the
    statically linked CUDA runtime and every C++ instance stay local, so two copies of the
    library in one process cannot bind to each other's internals."""
    import shutil
    import subprocess
    from learned_token_pruning_rmsnorm_b200 import _lib
    nm = shutil.which("nm")
    if nm is None:
        pytest.skip("no nm")
    r = subprocess.run([nm, "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True, check=True)
    names = sorted(line.split()[-1] for line in r.stdout.splitlines() if line.strip())
    assert names == _declared_functions()
