"""The C-ABI library loads here (no GPU needed), exports every symbol
include/dsa.h declares, and the ctypes structs match the C layout."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


def _declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"DSA_API\s+[\w\s\*]+?\b(dsa_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from sparse_attention_long_tcgen05_b200 import _build
    _build.build()
    from sparse_attention_long_tcgen05_b200 import dsa
    return dsa


def test_header_declares_the_abi():
    names = _declared_functions()
    for n in ["dsa_indexer_scores", "dsa_topk", "dsa_sparse_mqa_fwd", "dsa_forward",
              "dsa_workspace_size", "dsa_check_status", "dsa_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    so = ctypes.CDLL(lib.LIB_PATH)
    for name in _declared_functions():
        assert hasattr(so, name), name
    assert set(_declared_functions()) == set(lib.EXPORTED)


def test_status_strings_and_version(lib):
    assert lib.status_string(0) == "ok"
    assert "range" in lib.status_string(lib.DSA_ERR_DEVICE_BOUNDS)
    assert lib.LIB.dsa_version() >= 200


def test_workspace_size_host_logic(lib):
    """Workspace arithmetic needs no device: fused prefill keeps one bounded
    block of score rows (<= 80 MiB) plus the selection."""
    import torch
    L = 131072
    q = torch.empty(L, 64, 128, dtype=torch.uint8)
    k = torch.empty(L, 128, dtype=torch.uint8)
    w = torch.empty(L, 64)
    s = torch.empty(L)
    ind = lib.indexer_in(q, k, w, s, s)
    nbytes = lib.dsa_workspace_size(lib.DSA_OP_FORWARD, ind, None, 0, 0, 2048)
    idx_bytes = L * 2048 * 4
    assert idx_bytes < nbytes <= idx_bytes + (80 << 20) + 512
    assert lib.dsa_workspace_size(lib.DSA_OP_SPARSE_MQA) == 0
    # the score block: whole waves of 148 top-k CTAs within 80 MiB, or the
    # whole prefill when it fits
    for n in (4096, 32768, 65536, 131072):
        qn = torch.empty(n, 64, 128, dtype=torch.uint8)
        kn = torch.empty(n, 128, dtype=torch.uint8)
        sn = torch.empty(n)
        indn = lib.indexer_in(qn, kn, torch.empty(n, 64), sn, sn)
        sel = lib.dsa_workspace_size(lib.DSA_OP_SELECT, indn, None, 0, 0, 2048)
        rows = sel // (n * 4)
        assert sel - rows * n * 4 < 256 and rows * n * 4 <= (80 << 20)
        assert rows == n if n * n * 4 <= (80 << 20) else rows % 148 == 0
    with pytest.raises(lib.DsaError):
        lib.dsa_workspace_size(lib.DSA_OP_FORWARD, ind, None, 0, 0, 4096)   # k > 2048


def test_struct_layout_matches_c(lib):
    src = r"""
#include <stdio.h>
#include <stddef.h>
#include "dsa.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu %zu\n", sizeof(dsa_kv_layout),
         offsetof(dsa_kv_layout, block_table), offsetof(dsa_kv_layout, ld_block_table),
         offsetof(dsa_kv_layout, ctx_lens), offsetof(dsa_kv_layout, q_seq),
         offsetof(dsa_kv_layout, q_pos), offsetof(dsa_kv_layout, n_seq));
  printf("%zu %zu %zu %zu %zu %zu\n", sizeof(dsa_indexer_in), offsetof(dsa_indexer_in, q),
         offsetof(dsa_indexer_in, q_scale), offsetof(dsa_indexer_in, w),
         offsetof(dsa_indexer_in, ld_w), offsetof(dsa_indexer_in, kv));
  printf("%zu %zu %zu %zu %zu\n", sizeof(dsa_attn_in), offsetof(dsa_attn_in, scale),
         offsetof(dsa_attn_in, q), offsetof(dsa_attn_in, v), offsetof(dsa_attn_in, kv_layout));
  return 0;
}
"""
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "layout.c")
        exe = os.path.join(d, "layout")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        got = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()
    got = [int(x) for x in got]
    K, I, A = lib.KvLayout, lib.IndexerIn, lib.AttnIn
    want = [ctypes.sizeof(K), K.block_table.offset, K.ld_block_table.offset, K.ctx_lens.offset,
            K.q_seq.offset, K.q_pos.offset, K.n_seq.offset,
            ctypes.sizeof(I), I.q.offset, I.q_scale.offset, I.w.offset, I.ld_w.offset,
            I.kv.offset,
            ctypes.sizeof(A), A.scale.offset, A.q.offset, A.v.offset, A.kv_layout.offset]
    assert got == want


def test_product_never_reaches_the_oracle():
    """No file of the package (Python or CUDA) imports or includes the oracle."""
    pkg = os.path.join(ROOT, "sparse_attention_long_tcgen05_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle", text, re.M), f
                assert "dsa_oracle" not in text, f
