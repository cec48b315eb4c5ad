"""C-ABI checks that need no GPU: the library builds and loads, exports every function that
include/mla.h declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla.h")


@pytest.fixture(scope="module")
def M():
    from mla_latent_kv_37_b200 import build
    build.build()
    import mla_latent_kv_37_b200 as m
    return m


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_four_calls():
    names = _declared()
    for n in ("mla_cache_append", "mla_absorb_q", "mla_decode_attn", "mla_out_proj"):
        assert n in names


def test_library_exports_every_declared_symbol(M):
    out = subprocess.run(["nm", "-D", "--defined-only", M.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (mla_\w+)", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(M.LIB_PATH)
    for n in _declared():
        assert getattr(lib, n)


def _d(M, **kw):
    d = M.dims(4, 128, 7168)
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def test_layout_constants(M):
    import torch
    assert M.mla_cache_row_bytes(M.dims(1)) == 1152
    # 61 layers of one token: the 70,272 bytes the MLA pages print
    assert 61 * M.mla_cache_row_bytes(M.dims(1)) == 70272
    assert M.mla_cache_row_bytes(M.dims(1, 16, 1024, dtype=torch.float32)) == 2304
    assert M.mla_cache_row_bytes(_d(M, d_c=256)) == 0


@pytest.mark.parametrize("field,value", [("d_c", 256), ("d_rope", 32), ("d_nope", 64),
                                         ("d_v", 64), ("page_size", 32), ("n_heads", 24),
                                         ("n_heads", 256), ("d_model", 100), ("batch", 0),
                                         ("dtype", 7), ("rope_theta", 0.0), ("batch", 129)])
def test_unsupported_dims_rejected(M, field, value):
    d = _d(M, **{field: value})
    assert M.mla_workspace_size(d) == 0
    L = M.lib()
    fake = ctypes.c_void_p(0x10000)
    rc = L.mla_decode_attn(ctypes.byref(d), fake, None, fake, 10, fake, 4, fake, 0.0, 0, fake,
                           1 << 30, fake, None, None)
    assert rc == -2


def test_null_and_alignment_errors(M):
    d = _d(M)
    L = M.lib()
    f = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)  # 8-byte aligned only
    assert L.mla_decode_attn(None, f, None, f, 10, f, 4, f, 0.0, 0, f, 1 << 30, f, None, None) == -1
    assert L.mla_decode_attn(ctypes.byref(d), None, None, f, 10, f, 4, f, 0.0, 0, f, 1 << 30, f,
                             None, None) == -1
    assert L.mla_decode_attn(ctypes.byref(d), odd, None, f, 10, f, 4, f, 0.0, 0, f, 1 << 30, f,
                             None, None) == -3
    assert L.mla_decode_attn(ctypes.byref(d), f, None, f, 10, f, 4, f, 0.0, 0, None, 1 << 30, f,
                             None, None) == -4
    assert L.mla_decode_attn(ctypes.byref(d), f, None, f, 0, f, 4, f, 0.0, 0, f, 1 << 30, f, None,
                             None) == -5
    assert L.mla_decode_attn(ctypes.byref(d), f, None, f, 10, f, 4, f, -1.0, 0, f, 1 << 30, f,
                             None, None) == -5
    assert L.mla_cache_append(ctypes.byref(d), f, f, None, f, f, 4, f, 10, f, 1 << 30, None) == -1
    assert L.mla_absorb_q(ctypes.byref(d), f, f, f, f, f, None, None, 0, None) == -4
    assert L.mla_out_proj(ctypes.byref(d), f, f, f, None, None, f, 1 << 30, None) == -1
    assert L.mla_out_proj(ctypes.byref(d), f, f, None, None, None, f, 1 << 30, None) == -1


def test_query_remainder_arguments(M):
    # mla_decode_attn takes the query's rounding remainder on the bf16 path only; the
    # static-scratch entry point takes the bf16 query alone.  Both are host-side checks.
    import torch
    d = _d(M)
    L = M.lib()
    f = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    d32 = M.dims(4, 16, 1024, dtype=torch.float32)
    assert L.mla_decode_attn(ctypes.byref(d32), f, f, f, 10, f, 4, f, 0.0, 0, f, 1 << 30, f,
                             None, None) == -5
    assert L.mla_decode_attn(ctypes.byref(d), f, odd, f, 10, f, 4, f, 0.0, 0, f, 1 << 30, f,
                             None, None) == -3
    assert L.mla_decode_attn_static_scratch(ctypes.byref(d), f, f, f, 10, f, 4, f, 0.0, 0, f,
                                            None, None) == -5
    if not torch.cuda.is_available():  # the host checks pass; then the missing device shows
        rc = L.mla_decode_attn(ctypes.byref(d), f, f, f, 10, f, 4, f, 0.0, 0, f, 1 << 30, f,
                               None, None)
        assert rc in (-6, -7)


def test_split_count_and_page_bounds(M):
    # num_splits above 65536 and page counts whose token count overflows int32 are rejected
    # before any arithmetic on them
    d = _d(M)
    L = M.lib()
    f = ctypes.c_void_p(0x10000)
    assert M.mla_workspace_size(d, 65537) == 0
    assert M.mla_workspace_size(d, 65536) > 0
    for fn in (lambda *a: L.mla_decode_attn(*a[:10], f, 1 << 40, f, None, None),
               lambda *a: L.mla_decode_attn_static_scratch(*a, f, None, None)):
        assert fn(ctypes.byref(d), f, None, f, 10, f, 4, f, 0.0, 65537) == -5
        assert fn(ctypes.byref(d), f, None, f, 10, f, 1 << 25, f, 0.0, 0) == -5
        assert fn(ctypes.byref(d), f, None, f, 1 << 25, f, 4, f, 0.0, 0) == -5


def test_valid_call_without_gpu_fails_loudly(M):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    d = _d(M)
    f = ctypes.c_void_p(0x10000)
    rc = M.lib().mla_decode_attn(ctypes.byref(d), f, None, f, 10, f, 4, f, 0.0, 0, f, 1 << 30, f,
                                 None, None)
    assert rc in (-6, -7)


def test_workspace_size_is_positive_and_grows_with_splits(M):
    d = _d(M)
    a, b = M.mla_workspace_size(d, 8), M.mla_workspace_size(d, 200)
    assert 0 < a < b
    assert a % 256 == 0


def test_error_strings(M):
    L = M.lib()
    for code in (0, -1, -2, -3, -4, -5, -6, -7, 1, 4):
        assert L.mla_error_string(code)
    assert b"sm_100a" in L.mla_version()


def test_merge_partials_arguments(M):
    d = _d(M)
    L = M.lib()
    f = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    assert L.mla_merge_partials(ctypes.byref(d), 0, f, f, f, None, None) == -5
    assert L.mla_merge_partials(ctypes.byref(d), 2, None, f, f, None, None) == -1
    assert L.mla_merge_partials(ctypes.byref(d), 2, odd, f, f, None, None) == -3
    assert L.mla_merge_partials(ctypes.byref(_d(M, d_c=256)), 2, f, f, f, None, None) == -2


def test_folded_mode_arguments(M):
    """The folded execution mode is bf16 only and checks its pointers on the host."""
    import torch
    d = _d(M)
    d32 = M.dims(4, 16, 1024, dtype=torch.float32)
    L = M.lib()
    f = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    ws = ctypes.c_void_p(0x100000)
    big = ctypes.c_size_t(1 << 40)
    # folding: fp32 rejected; nothing to fold; an output without its inputs; misaligned
    assert L.mla_fold_weights(ctypes.byref(d32), f, f, f, f, f, f, None) == -5
    assert L.mla_fold_weights(ctypes.byref(d), f, f, f, f, None, None, None) == -1
    assert L.mla_fold_weights(ctypes.byref(d), None, f, None, None, f, None, None) == -1
    assert L.mla_fold_weights(ctypes.byref(d), None, None, f, None, None, f, None) == -1
    assert L.mla_fold_weights(ctypes.byref(d), odd, f, None, None, f, None, None) == -3
    assert L.mla_fold_weights(ctypes.byref(_d(M, d_c=256)), f, f, f, f, f, f, None) == -2
    # folded append + query
    args = [f, f, f, f, f, f, 4, f, 8, f, None, ws, big, None]
    assert L.mla_append_absorb_folded(ctypes.byref(d32), *args) == -5
    bad = list(args)
    bad[3] = None  # w_qf
    assert L.mla_append_absorb_folded(ctypes.byref(d), *bad) == -1
    bad = list(args)
    bad[3] = odd
    assert L.mla_append_absorb_folded(ctypes.byref(d), *bad) == -3
    bad = list(args)
    bad[6] = 0  # max_pages
    assert L.mla_append_absorb_folded(ctypes.byref(d), *bad) == -5
    bad = list(args)
    bad[11] = None  # workspace
    assert L.mla_append_absorb_folded(ctypes.byref(d), *bad) == -4
    # folded output product
    assert L.mla_out_proj_folded(ctypes.byref(d32), f, f, f, ws, big, None) == -5
    assert L.mla_out_proj_folded(ctypes.byref(d), f, None, f, ws, big, None) == -1
    assert L.mla_out_proj_folded(ctypes.byref(d), f, f, odd, ws, big, None) == -3
    assert L.mla_out_proj_folded(ctypes.byref(d), f, f, f, None, big, None) == -4


def test_step_executor_arguments(M):
    """The native step executor's host checks, before it touches CUDA."""
    d = _d(M)
    L = M.lib()
    f = ctypes.c_void_p(0x10000)
    ws = ctypes.c_void_p(0x100000)
    big = ctypes.c_size_t(1 << 40)
    assert L.mla_step_workspace_size(ctypes.byref(d), 0, 0) == 0
    assert L.mla_step_workspace_size(ctypes.byref(d), 2, 0) > L.mla_step_workspace_size(
        ctypes.byref(d), 1, 0) > L.mla_workspace_size(ctypes.byref(d), 0)
    lay = (M.mla_layer * 2)()
    for i in range(2):
        lay[i] = M.mla_layer(0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 8,
                             0x10000, 4)
    assert L.mla_decode_step_host(ctypes.byref(d), 0, lay, f, f, f, f, 0, ws, big, None) == -5
    assert L.mla_decode_step_host(ctypes.byref(d), 2, None, f, f, f, f, 0, ws, big, None) == -1
    assert L.mla_decode_step_host(ctypes.byref(d), 2, lay, None, f, f, f, 0, ws, big, None) == -1
    assert L.mla_decode_step_host(ctypes.byref(d), 2, lay, f, f, f, f, 0, None, big, None) == -4
    assert L.mla_decode_step_host(ctypes.byref(d), 2, lay, f, f, f, f, 0,
                                  ctypes.c_void_p(0x100010), big, None) == -3
    assert L.mla_decode_step_host(ctypes.byref(d), 2, lay, f, f, f, f, 0, ws,
                                  ctypes.c_size_t(1024), None) == -4
    lay[1] = M.mla_layer(0x10000, 0x10000, 0x10000, 0x10000, 0x10000, None, 0x10000, 8,
                         0x10000, 4)
    assert L.mla_decode_step_host(ctypes.byref(d), 2, lay, f, f, f, f, 0, ws, big, None) == -1
    # an E4M3 layer (w_q_scale given) needs every row scale
    lay[1] = M.mla_layer(0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 8,
                         0x10000, 4, 0x10000, None, 0x10000, 0x10000)
    assert L.mla_decode_step_host(ctypes.byref(d), 2, lay, f, f, f, f, 0, ws, big, None) == -1



def test_e4m3_weight_arguments(M):
    """The E4M3-weight calls check their arguments on the host, before any device work: code
    widths that are not whole 128-column tiles, missing or misaligned pointers, the fp32
    path, batches above 128 and d_model not a multiple of 128."""
    import torch
    d = _d(M)
    d32 = M.dims(4, 16, 1024, dtype=torch.float32)
    L = M.lib()
    f = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    ws = ctypes.c_void_p(0x100000)
    big = ctypes.c_size_t(1 << 40)
    # quantization: cols a positive multiple of 128, pointers present and aligned
    assert L.mla_quantize_weights_fp8(f, 8, 64, f, f, None) == -5
    assert L.mla_quantize_weights_fp8(f, 0, 128, f, f, None) == -5
    assert L.mla_quantize_weights_fp8(None, 8, 128, f, f, None) == -1
    assert L.mla_quantize_weights_fp8(f, 8, 128, odd, f, None) == -3
    # append + absorb with E4M3 W_DKV, W_KR, W_Q
    args = [f, f, f, f, f, f, f, f, f, f, 4, f, 8, f, None, ws, big, None]
    assert L.mla_append_absorb_fp8(ctypes.byref(d32), *args) == -5
    assert L.mla_append_absorb_fp8(ctypes.byref(M.dims(129, 16, 1024)), *args) == -2
    assert L.mla_append_absorb_fp8(ctypes.byref(M.dims(4, 16, 1088)), *args) == -2
    for i, code in ((1, -1), (6, -1), (7, -1), (13, -1)):  # codes, scale, w_uk, q_cat
        bad = list(args)
        bad[i] = None
        assert L.mla_append_absorb_fp8(ctypes.byref(d), *bad) == code
    bad = list(args)
    bad[5] = odd  # W_Q codes
    assert L.mla_append_absorb_fp8(ctypes.byref(d), *bad) == -3
    bad = list(args)
    bad[15] = None  # workspace
    assert L.mla_append_absorb_fp8(ctypes.byref(d), *bad) == -4
    # output projection with E4M3 W_O
    oargs = [f, f, f, f, None, f, ws, big, None]
    assert L.mla_out_proj_fp8(ctypes.byref(d32), *oargs) == -5
    assert L.mla_out_proj_fp8(ctypes.byref(M.dims(129, 16, 1024)), *oargs) == -2
    bad = list(oargs)
    bad[5] = None  # out
    assert L.mla_out_proj_fp8(ctypes.byref(d), *bad) == -1
    bad = list(oargs)
    bad[2] = odd  # W_O codes
    assert L.mla_out_proj_fp8(ctypes.byref(d), *bad) == -3


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "mla.h"

int main(void) {
  mla_dims d;
  memset(&d, 0, sizeof d);
  d.batch = 4;
  d.n_heads = 128;
  d.d_model = 7168;
  d.d_c = 512;
  d.d_rope = 64;
  d.d_nope = 128;
  d.d_v = 128;
  d.page_size = 64;
  d.dtype = MLA_BF16;
  d.rope_theta = 10000.0f;
  printf("version %s\n", mla_version());
  printf("row_bytes %lld\n", (long long)mla_cache_row_bytes(&d));
  printf("workspace_nonzero %d\n", mla_workspace_size(&d, 0) > 0);
  printf("null_args %d\n", mla_decode_attn(&d, NULL, NULL, NULL, 1, NULL, 1, NULL, 0.f, 0, NULL,
                                          0, NULL, NULL, NULL));
  printf("error_string %s\n", mla_error_string(MLA_ERR_NULL_ARG));
  return 0;
}
"""


def test_header_is_plain_c_and_links(M, tmp_path):
    """include/mla.h compiles as strict C99 with every warning an error, and a C program links
    against the library and calls it: the boundary needs neither C++ nor Python."""
    import os
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(C_PROGRAM)
    lib_dir = os.path.dirname(M.LIB_PATH)
    exe = tmp_path / "abi"
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-I", os.path.dirname(HEADER), str(src), "-L", lib_dir, "-lmla_b200",
                        "-Wl,-rpath," + lib_dir, "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    lines = dict(line.split(" ", 1) for line in out.stdout.strip().splitlines())
    assert lines["row_bytes"] == "1152"
    assert lines["workspace_nonzero"] == "1"
    assert lines["null_args"] == "-1"
    assert lines["version"]
