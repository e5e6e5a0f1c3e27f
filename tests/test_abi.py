"""The C-ABI library loads, exports every declared symbol, and its descriptor
structs match the binding.  No compute call is made here (CPU-only)."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


def _lib():
    from long_context_sparse_04_b200 import build
    build.build()
    from long_context_sparse_04_b200 import _native as N
    return N


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(dsa_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla_fwd", "dsa_decode_step",
              "dsa_forward", "dsa_workspace_size", "dsa_read_device_status"):
        assert n in names


def test_library_exports_every_declared_symbol():
    N = _lib()
    for name in declared_functions():
        assert hasattr(N.LIB, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", N.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (dsa_\w+)", out))
    assert set(declared_functions()) <= exported


def test_struct_layout_matches_c_compiler():
    N = _lib()
    prog = r'''
#include <stdio.h>
#include <stddef.h>
#include "dsa.h"
int main(void) {
  printf("%zu %zu %zu\n", sizeof(dsa_dims), sizeof(dsa_rows), sizeof(dsa_cache));
  printf("%zu %zu %zu %zu\n", offsetof(dsa_dims, sm_scale), offsetof(dsa_rows, row_klen),
         offsetof(dsa_rows, q_group), offsetof(dsa_cache, num_tokens));
  return 0;
}
'''
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        open(c, "w").write(prog)
        exe = os.path.join(d, "t")
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        a, b = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")[:2]
    assert list(map(int, a.split())) == [ctypes.sizeof(N.dsa_dims), ctypes.sizeof(N.dsa_rows),
                                         ctypes.sizeof(N.dsa_cache)]
    assert list(map(int, b.split())) == [N.dsa_dims.sm_scale.offset, N.dsa_rows.row_klen.offset,
                                         N.dsa_rows.q_group.offset, N.dsa_cache.num_tokens.offset]


def _dims(N, **kw):
    d = dict(n_idx_heads=64, d_idx=128, n_heads=128, d_c=512, d_r=64, topk=2048,
             idx_dtype=N.DSA_FP8_E4M3, mla_dtype=N.DSA_BF16, sm_scale=1 / 24, algo=0)
    d.update(kw)
    return N.dsa_dims(**d)


def test_status_strings_and_version():
    N = _lib()
    assert N.LIB.dsa_status_string(0) == b"DSA_OK"
    assert N.LIB.dsa_status_string(5) == b"DSA_ERR_TIMEOUT"
    assert N.LIB.dsa_version() >= 100


def test_workspace_size_plans():
    N = _lib()
    fake = ctypes.c_void_p(256)
    rows = N.dsa_rows(num_rows=32, row_seq=fake, row_klen=fake, max_klen=131071, q_group=2)
    dims = _dims(N)
    dec = N.dsa_workspace_size(dims, rows, N.DSA_OP_DECODE_STEP)
    # scores buffer T x round_up(max_klen,128) fp32 + indices must fit
    assert dec >= 32 * 131072 * 4 + 32 * 2048 * 4
    assert N.dsa_workspace_size(dims, rows, N.DSA_OP_TOPK) >= 256
    bad = _dims(N, topk=4096)
    assert N.dsa_workspace_size(bad, rows, N.DSA_OP_DECODE_STEP) == 0
    rows_bad = N.dsa_rows(num_rows=32, row_seq=fake, row_klen=fake, max_klen=10, q_group=3)
    assert N.dsa_workspace_size(dims, rows_bad, N.DSA_OP_TOPK) == 0


def test_cache_append_and_projection_workspace_sizes():
    N = _lib()
    assert N.dsa_workspace_size(_dims(N), None, N.DSA_OP_CACHE_APPEND) == 256
    p = N.dsa_proj_dims(n_heads=128, d_c=512, d_v=128, d_model=7168)
    assert N.dsa_output_projection_ws_size(p, 0) == 256          # no rows: status block only
    # a small batch splits K: status block + fp32 partials [splits, T, d_model]
    dec = N.dsa_output_projection_ws_size(p, 32)
    assert dec > 256 and (dec - 256) % (32 * 7168 * 4) == 0 and dec - 256 <= 16 * 32 * 7168 * 4
    assert N.dsa_output_projection_ws_size(p, 65536) == 256      # enough tiles: no split
    for bad in (dict(d_c=100), dict(d_v=48), dict(d_v=512), dict(d_model=100), dict(n_heads=0)):
        kw = dict(n_heads=128, d_c=512, d_v=128, d_model=7168)
        kw.update(bad)
        assert N.dsa_output_projection_ws_size(N.dsa_proj_dims(**kw), 8) == 0, bad


def test_argument_errors_are_reported_before_any_cuda_call():
    N = _lib()
    fake = ctypes.c_void_p(1 << 20)
    rows = N.dsa_rows(num_rows=4, row_seq=fake, row_klen=fake, max_klen=100, q_group=1)
    cache = N.dsa_cache(latent=fake, idx_k=fake, idx_k_scale=fake, seq_start=None,
                        block_table=None, page_size=0, max_pages_per_seq=0, num_seqs=1,
                        num_tokens=100)
    dims = _dims(N)
    st = N.dsa_indexer_scores(None, rows, cache, fake, fake, fake, fake, 128, fake, 1 << 20, None,
                              check=False)
    assert st == N.DSA_ERR_INVALID_ARG
    st = N.dsa_indexer_scores(dims, rows, cache, fake, fake, fake, fake, 64, fake, 1 << 20, None,
                              check=False)
    assert st == N.DSA_ERR_INVALID_ARG          # ld_scores < max_klen
    st = N.dsa_topk(dims, rows, fake, 128, fake, None, 0, None, check=False)
    assert st == N.DSA_ERR_WORKSPACE
    st = N.dsa_topk(dims, rows, fake, 128, fake, ctypes.c_void_p(1 << 20 | 8), 4096, None, check=False)
    assert st == N.DSA_ERR_WORKSPACE            # misaligned workspace
    st = N.dsa_topk(_dims(N, topk=0), rows, fake, 128, fake, fake, 4096, None, check=False)
    assert st == N.DSA_ERR_INVALID_ARG
    mis = ctypes.c_void_p((1 << 20) + 4)
    st = N.dsa_sparse_mla_fwd(dims, rows, cache, mis, fake, fake, None, fake, 1 << 24, None,
                              check=False)
    assert st == N.DSA_ERR_INVALID_ARG          # misaligned q
    paged = N.dsa_cache(latent=fake, idx_k=fake, idx_k_scale=fake, seq_start=None, block_table=fake,
                        page_size=64, max_pages_per_seq=4, num_seqs=1, num_tokens=100)
    st = N.dsa_decode_step(dims, rows, paged, fake, fake, fake, fake, fake, None, None, None, fake,
                           1 << 30, None, check=False)
    assert st == N.DSA_ERR_INVALID_ARG          # num_tokens not a whole number of pages
    with pytest.raises(N.DSAError):
        N.dsa_topk(_dims(N, topk=0), rows, fake, 128, fake, fake, 4096, None)


def test_fault_injection_rejects_unknown_bits():
    # host-side argument check only: no device work
    N = _lib()
    assert N.dsa_set_fault_injection(0, 0x80, check=False) == N.DSA_ERR_INVALID_ARG
    assert N.dsa_set_fault_injection(0, 0) == N.DSA_OK
