"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function declared in include/tri.h, and rejects bad arguments before
touching the device (nothing here launches a kernel)."""
import ctypes
import os
import subprocess

import pytest

from bit_mixed_precision_tri_b200 import _lib

FAKE = 1 << 20        # a non-null, 256-byte-aligned address that is never dereferenced


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(_lib.LIB_PATH):
        from bit_mixed_precision_tri_b200 import build
        build.build()
    return _lib.lib()


def test_exports_every_declared_symbol(L):
    declared = _lib.declared_symbols()
    assert len(declared) >= 13
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in declared:
        assert name in exported, name
        assert hasattr(L, name)
    assert set(_lib.SIGNATURES) == set(declared)


def test_status_strings_and_version(L):
    assert L.tri_version() >= 100
    for s in range(11):
        assert L.tri_status_string(s)
    assert L.tri_status_string(12345) == b"unknown status"


def test_gemm_argument_validation(L):
    g = L.tri_gemm
    ok = dict(fmt=2, path=0, X=FAKE, qs=FAKE, d=FAKE, Y=FAKE, M=1, N=8, K=256)

    def call(**kw):
        a = dict(ok, **kw)
        return g(a["fmt"], a["path"], a["X"], a["qs"], a["d"], a["Y"], a["M"], a["N"], a["K"],
                 None, 0, None)

    assert call(fmt=3) == 1
    assert call(path=9) == 1
    assert call(X=None) == 1
    assert call(M=0) == 2
    assert call(N=0) == 2
    assert call(K=255) == 2
    assert call(K=300) == 2
    assert call(K=0) == 2
    assert call(M=1 << 31) == 2
    assert call(X=FAKE + 8) == 3
    assert call(Y=FAKE + 2) == 3
    assert call(qs=FAKE + 4) == 3                   # TQ2 planes need 16-byte alignment
    assert call(fmt=1, qs=FAKE + 4, X=FAKE + 8) == 3  # X still misaligned


def test_pack_unpack_and_absmean_validation(L):
    assert L.tri_pack_tq2(None, 4, 256, FAKE, 1, FAKE, FAKE, None, None) == 1
    assert L.tri_pack_tq2(FAKE, 4, 256, FAKE, 3, FAKE, FAKE, None, None) == 1   # n_scales
    assert L.tri_pack_tq1(FAKE, 4, 100, FAKE, 1, FAKE, FAKE, None, None) == 2
    assert L.tri_pack_tq2(FAKE + 1, 4, 256, FAKE, 1, FAKE, FAKE, None, None) == 3
    assert L.tri_unpack(7, FAKE, 4, 256, FAKE, None, None) == 1
    assert L.tri_unpack(2, FAKE, 4, 512 + 1, FAKE, None, None) == 2
    ws = L.tri_absmean_workspace_bytes(4, 256)
    assert ws >= 256 * 8
    assert L.tri_absmean(FAKE, 4, 256, -1.0, FAKE, FAKE, ws, None) == 1          # eps < 0
    assert L.tri_absmean(FAKE, 4, 256, 1e-6, FAKE, FAKE, ws - 1, None) == 8      # workspace
    assert L.tri_absmean(FAKE, 4, 256, 1e-6, FAKE, None, ws, None) == 8
    assert L.tri_ternarize(FAKE, 4, 256, 1e-6, None, FAKE, FAKE, ws, None) == 1


def test_auto_path_and_workspace_query(L):
    assert L.tri_gemm_auto_path(2, 0, 8, 256) == -1
    assert L.tri_gemm_auto_path(5, 1, 8, 256) == -1
    for fmt in (1, 2):
        for M in (1, 16, 64, 256):
            p = L.tri_gemm_auto_path(fmt, M, 4096, 4096)
            assert p in (1, 2, 3, 4)
            assert L.tri_gemm_workspace_bytes(fmt, M, 4096, 4096) >= 256


def test_wait_status_entry_points_reject_bad_arguments(L):
    assert L.tri_wait_status(None, 1, None) == 1                       # null code pointer
    assert L.tri_selftest_wait_timeout(2, FAKE, None) == 1             # no such wait
    assert L.tri_selftest_wait_timeout(-1, FAKE, None) == 1
    assert L.tri_selftest_wait_timeout(0, None, None) == 1             # null scratch
    assert L.tri_selftest_wait_timeout(1, FAKE + 4, None) == 3         # scratch not 8-byte aligned


def test_decode_step_entry_points_validate_before_the_device(L):
    P = FAKE
    # tri_rmsnorm: nulls, eps, aliasing, shape, alignment
    assert L.tri_rmsnorm(None, None, P, None, P, 2, 64, 1e-5, None) == 1
    assert L.tri_rmsnorm(P, P, P, None, P, 2, 64, 1e-5, None) == 1            # residual needs h_out
    assert L.tri_rmsnorm(P, P + 256, P, P, P, 2, 64, 1e-5, None) == 1         # h_out aliases x
    assert L.tri_rmsnorm(P, None, P, None, P, 2, 64, -1.0, None) == 1
    assert L.tri_rmsnorm(P, None, P, None, P, 2, 60, 1e-5, None) == 2          # D % 8
    assert L.tri_rmsnorm(P, None, P, None, P, 0, 64, 1e-5, None) == 2
    assert L.tri_rmsnorm(P + 8, None, P, None, P, 2, 64, 1e-5, None) == 3
    # tri_rope_table
    assert L.tri_rope_table(None, 16, 128, 5e5, None) == 1
    assert L.tri_rope_table(P, 16, 128, 1.0, None) == 1                        # theta must exceed 1
    assert L.tri_rope_table(P, 16, 64, 5e5, None) == 2                         # head dim 128 only
    assert L.tri_rope_table(P, 0, 128, 5e5, None) == 2
    assert L.tri_rope_table(P + 4, 16, 128, 5e5, None) == 3
    # tri_qknorm_rope
    args = [P, P, P, P, P, P, P, P]
    assert L.tri_qknorm_rope(*([None] + args[1:]), 1, 8, 2, 16, 1e-5, None) == 1
    assert L.tri_qknorm_rope(*args, 1, 8, 3, 16, 1e-5, None) == 2             # H % Hkv
    assert L.tri_qknorm_rope(*args, 1, 8, 2, 0, 1e-5, None) == 2
    assert L.tri_qknorm_rope(*([P + 8] + args[1:]), 1, 8, 2, 16, 1e-5, None) == 3
    assert L.tri_qknorm_rope(*(args[:1] + [P + 2] + args[2:]), 1, 8, 2, 16, 1e-5, None) == 3   # pos
    # tri_attention_decode and its workspace query
    assert L.tri_attention_decode_workspace_bytes(1, 64, 8, 4096) > 0
    assert L.tri_attention_decode_workspace_bytes(1, 64, 4, 4096) == 0         # 16 query heads per group
    assert L.tri_attention_decode_workspace_bytes(1, 64, 8, 0) == 0
    assert L.tri_attention_decode(None, P, P, P, P, 1, 64, 8, 4096, 4096, P, 1 << 20, None) == 1
    assert L.tri_attention_decode(P, P, P, P, P, 1, 64, 8, 4096, 4097, P, 1 << 20, None) == 2  # max_len > Lmax
    assert L.tri_attention_decode(P + 8, P, P, P, P, 1, 64, 8, 4096, 4096, P, 1 << 20, None) == 3   # q
    assert L.tri_attention_decode(P, P, P, P + 2, P, 1, 64, 8, 4096, 4096, P, 1 << 20, None) == 3   # pos


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "tri.h"

/* A plain C99 caller: the header must compile as C, every declared entry
 * point must link, and the calls that touch no device must answer. */
int main(void) {
  if (tri_version() < 100) return 1;
  if (strcmp(tri_status_string(TRI_OK), "ok") != 0) return 2;
  if (tri_gemm_auto_path(TRI_TQ2, 0, 8, 256) != -1) return 3;
  if (tri_gemm(TRI_TQ2, TRI_PATH_AUTO, NULL, NULL, NULL, NULL, 1, 8, 256, NULL, 0, NULL)
      != TRI_ERR_INVALID_ARG) return 4;
  if (tri_gemm_swiglu(TRI_TQ2, TRI_PATH_AUTO, NULL, NULL, NULL, NULL, 1, 8, 256, NULL, 0, NULL)
      != TRI_ERR_INVALID_ARG) return 5;
  if (tri_wait_status(NULL, 1, NULL) != TRI_ERR_INVALID_ARG) return 6;
  if (tri_selftest_wait_timeout(7, NULL, NULL) != TRI_ERR_INVALID_ARG) return 7;
  if (tri_gemm_swiglu_workspace_bytes(TRI_TQ2, 4, 12, 256) != 0) return 8;   /* F % 8 != 0 */
  /* every other entry point is referenced so that the link resolves it */
  void* fns[] = {(void*)tri_last_cuda_error, (void*)tri_absmean_workspace_bytes, (void*)tri_absmean,
                 (void*)tri_ternarize, (void*)tri_pack_tq2, (void*)tri_pack_tq1, (void*)tri_unpack,
                 (void*)tri_gemm_workspace_bytes, (void*)tri_gemm_tq2, (void*)tri_gemm_tq1,
                 (void*)tri_gemm_tq2_noalloc, (void*)tri_gemm_tq2_noalloc_fits};
  for (unsigned i = 0; i < sizeof(fns) / sizeof(fns[0]); ++i)
    if (!fns[i]) return 9;
  printf("c-abi ok\n");
  return 0;
}
"""


def test_header_compiles_as_c_and_links(L, tmp_path):
    """The boundary is usable from plain C (no C++ or torch types): a C99
    program includes include/tri.h, links the in-tree library and calls the
    entry points that need no device."""
    import shutil
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi_check.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi_check"
    libdir = os.path.dirname(_lib.LIB_PATH)
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(_lib.HEADER), str(src),
                        "-o", str(exe), "-L", libdir, "-l:" + os.path.basename(_lib.LIB_PATH),
                        "-Wl,-rpath," + libdir], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert "c-abi ok" in r.stdout
