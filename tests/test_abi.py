"""CPU-side checks of the C ABI: the library loads, exports every symbol the header declares,
and rejects invalid arguments on the host before touching the GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msa.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(msa_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def msa():
    import long_context_doc_b200 as m
    return m


def test_header_declarations_are_exported(msa):
    names = _declared()
    assert len(names) >= 16
    for n in names:
        assert hasattr(msa.lib, n), f"{n} declared in msa.h but not exported"
    assert set(names) == set(msa.SYMBOLS)
    # nothing else with the public prefix is exported
    out = os.popen(f"nm -D --defined-only {msa.LIB_PATH}").read()
    exported = set(re.findall(r"\bT (msa_[a-z_0-9]+)\b", out))
    assert exported == set(names), exported ^ set(names)


def test_status_strings_and_version(msa):
    assert msa.lib.msa_status_string(0) == b"MSA_OK"
    assert msa.lib.msa_status_string(5) == b"MSA_ERR_TIMEOUT"
    assert msa.lib.msa_version() >> 16 == 1


def test_count_chunks_matches_layout(msa):
    import synth
    lens = np.array([1, 64, 65, 500, 0, 128])
    off = np.concatenate([[0], np.cumsum(lens)])
    coff = synth.chunk_offsets_from_lengths(lens, 64)
    assert msa.msa_count_chunks(off, 64) == coff[-1]
    assert msa.msa_count_chunks(np.array([0, 5, 3]), 64) == -1
    assert msa.msa_count_chunks(np.array([1, 5]), 64) == -1


def _call_encode(msa, d=64, dtype=0, chunk=64, n_chunks=None, h_kv=2):
    off = np.array([0, 100, 228], np.int64)
    nc = msa.msa_count_chunks(off, chunk) if n_chunks is None else n_chunks
    fake = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    return msa.lib.msa_encode_pool(fake, fake, fake, 228, off.ctypes.data, fake, 2, chunk, h_kv,
                                   d, dtype, 1e6, fake, fake, fake, None, fake, nc, None)


def test_encode_rejects_bad_arguments_on_host(msa):
    assert _call_encode(msa, d=96) == 2             # UNSUPPORTED head dim
    assert _call_encode(msa, dtype=7) == 2           # UNSUPPORTED dtype
    assert _call_encode(msa, n_chunks=5) == 1        # INVALID_ARG: inconsistent chunk count
    assert _call_encode(msa, chunk=0) == 1
    assert _call_encode(msa, h_kv=3) == 2            # encode needs a power-of-two h_kv
    assert b"n_chunks" in msa.lib.msa_last_error() or True


def test_route_rejects_bad_arguments_on_host(msa):
    fake = ctypes.c_void_p(256)
    r = msa.lib.msa_route_topk(fake, 2, 1, 8, fake, fake, None, fake, 10, 80, 8, 128, 1, 11, None, fake,
                               fake, None, fake, 1 << 20, None)
    assert r == 1 and b"k 11" in msa.lib.msa_last_error()          # k > n_docs
    r = msa.lib.msa_route_topk(fake, 2, 1, 8, fake, fake, None, fake, 100, 800, 8, 128, 1, 33, None,
                               fake, fake, None, fake, 1 << 20, None)
    assert r == 2                                                   # k > 32 unsupported
    r = msa.lib.msa_route_topk(fake, 2, 1, 6, fake, fake, None, fake, 100, 800, 8, 128, 1, 4, None, fake,
                               fake, None, fake, 1 << 20, None)
    assert r == 1                                                   # h_qr % h_kv
    r = msa.lib.msa_route_topk(fake, 1, 64, 8, fake, fake, None, fake, 100, 800, 8, 128, 1, 4, None,
                               fake, fake, None, fake, 1 << 20, None)
    assert r == 1                                                   # long query needs Kbar_r_hat
    r = msa.lib.msa_route_topk(fake, 1, 64, 8, fake, fake, fake, fake, 100, 800, 8, 128, 0, 4, None,
                               fake, fake, None, fake, 1 << 20, None)
    assert r == 2                                                   # long fp32 query
    r = msa.lib.msa_route_topk(fake, 1, 300, 8, fake, fake, fake, fake, 100, 800, 8, 128, 1, 4,
                               None, fake, fake, None, fake, 1 << 20, None)
    assert r == 2                                                   # T > 256


def test_attend_and_gather_reject_bad_arguments_on_host(msa):
    fake = ctypes.c_void_p(256)
    # T > L_loc
    r = msa.lib.msa_sparse_attend(fake, 1, 4, 8, fake, fake, 2, fake, fake, fake, 8, 2, 64, 0, 4,
                                  1e6, 0.0, fake, fake, 1 << 20, None)
    assert r == 1
    # h_q not a multiple of h_kv
    r = msa.lib.msa_sparse_attend(fake, 1, 1, 6, fake, fake, 2, fake, fake, fake, 8, 4, 64, 0, 4,
                                  1e6, 0.0, fake, fake, 1 << 20, None)
    assert r == 1
    # gather without a workspace
    r = msa.lib.msa_gather(fake, 1, 4, fake, 10, fake, fake, 2, 64, 0, 32, fake, fake, fake, fake,
                           None, 0, None)
    assert r == 3


def test_fetch_finish_requires_begin(msa):
    r = msa.lib.msa_fetch_finish(None, None, 0, None, None, 8, 128, 1, 16, None, None, None, None, 0)
    assert r == 1


def test_attend_fast_paths_check_their_workspace_on_host(msa):
    """bf16 d=128 decode (<= 8 rows per KV head) and long-query (>= 64 rows) shapes take their
    own kernels; each refuses a workspace smaller than its plan before touching the device."""
    fake = ctypes.c_void_p(256)
    for T, L in ((1, 2048), (64, 300)):  # decode kernel, tensor-core kernel
        need = msa.msa_sparse_attend_workspace(2, T, 32, 8, 128, 128, L)
        assert need > 256
        r = msa.lib.msa_sparse_attend(fake, 2, T, 32, fake, fake, L, fake, fake, fake, 128, 8, 128,
                                      1, 16, 1e6, 0.0, fake, fake, 256, None)
        assert r == 3, (T, r)


def test_assemble_local_rejects_bad_arguments_on_host(msa):
    fake = ctypes.c_void_p(256)
    ws = ctypes.c_void_p(512)
    # more than 1024 segments per query
    r = msa.lib.msa_assemble_local(2, 1025, fake, fake, fake, fake, fake, 4, 8, 128, 1, 10, fake,
                                   fake, ws, 256, None)
    assert r == 1
    # L_loc shorter than the query rows
    r = msa.lib.msa_assemble_local(2, 3, fake, fake, fake, fake, fake, 8, 8, 128, 1, 4, fake, fake,
                                   ws, 256, None)
    assert r == 1
    # no workspace
    r = msa.lib.msa_assemble_local(2, 3, fake, fake, fake, fake, fake, 4, 8, 128, 1, 10, fake, fake,
                                   None, 0, None)
    assert r == 3
    # missing output
    r = msa.lib.msa_assemble_local(2, 3, fake, fake, fake, fake, fake, 4, 8, 128, 1, 10, None, fake,
                                   ws, 256, None)
    assert r == 1


def test_generation_entry_points_reject_bad_arguments_on_host(msa):
    fake = ctypes.c_void_p(256)
    ws = ctypes.c_void_p(512)
    # kv_append: more new rows than the cache holds, no workspace, missing length, misaligned
    r = msa.lib.msa_kv_append(fake, fake, 2, 8, fake, fake, fake, 9, 8, 128, 1, 0, 0.0, ws, 256,
                              None)
    assert r == 1
    r = msa.lib.msa_kv_append(fake, fake, 2, 8, fake, fake, fake, 1, 8, 128, 1, 0, 0.0, None, 0,
                              None)
    assert r == 3
    r = msa.lib.msa_kv_append(fake, fake, 2, 8, None, fake, fake, 1, 8, 128, 1, 0, 0.0, ws, 256,
                              None)
    assert r == 1
    r = msa.lib.msa_kv_append(fake, fake, 2, 8, fake, fake, fake, 1, 8, 128, 1, -1, 1e6, ws, 256,
                              None)  # negative pos0
    assert r == 1
    r = msa.lib.msa_kv_append(fake, ctypes.c_void_p(264), 2, 8, fake, fake, fake, 1, 8, 128, 1,
                              0, 0.0, ws, 256, None)
    assert r == 1
    need = msa.msa_decode_step_workspace(4, 1, 32, 8, 128, 128, 4096)
    assert need > 256

    def step(dtype=1, h_q=32, h_kv=8, d=128, T=1, cap=4096, ws_bytes=need, L=fake):
        return msa.lib.msa_decode_step(fake, fake, fake, 4, T, h_q, fake, fake, cap, L, fake,
                                       fake, fake, 128, h_kv, d, dtype, 16, 1e6, 0.0, fake, ws,
                                       ws_bytes, None)
    assert step(dtype=0) == 2           # fp32: no decode kernel
    assert step(T=3) == 2               # 12 query rows per KV head
    assert step(h_kv=3, h_q=30) == 2    # 3 KV heads
    assert step(cap=0) == 1             # capacity below T
    assert step(ws_bytes=need - 1) == 3
    assert step(L=None) == 1            # no device length


def test_encode_hidden_rejects_bad_arguments_on_host(msa):
    import numpy as np
    fake = ctypes.c_void_p(256)
    off = np.array([0, 70, 80], np.int64)
    ws_bytes = msa.msa_encode_hidden_workspace(3)
    assert ws_bytes >= 256 + 3 * 12
    ws = ctypes.c_void_p(512)

    def call(D=256, chunk=64, h_kv=2, d=128, dtype=1, n_chunks=3, wsb=ws_bytes, offs=off):
        return msa.lib.msa_encode_hidden(fake, int(offs[-1]), D, fake, fake, fake,
                                         offs.ctypes.data, len(offs) - 1, chunk, h_kv, d, dtype,
                                         1e6, fake, fake, fake, fake, n_chunks, ws, wsb, None)
    assert call(dtype=0) == 2          # fp32
    assert call(chunk=32) == 2         # chunk must be 64
    assert call(h_kv=3) == 2           # odd KV heads
    assert call(D=100) == 2            # hidden size not a multiple of 64
    assert call(n_chunks=4) == 1       # inconsistent with the offsets
    assert call(offs=np.array([0, 70, 60], np.int64)) == 1  # decreasing offsets
    assert call(wsb=ws_bytes - 1) == 3


C_CALLER = r"""
/* A plain C11 caller of the boundary: header compiled as C, library linked as a C library. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>
#include "msa.h"

static int fail(const char* what) { fprintf(stderr, "FAIL %s\n", what); return 1; }

int main(void) {
  if ((msa_version() >> 16) != 1) return fail("version");
  if (strcmp(msa_status_string(MSA_OK), "MSA_OK") != 0) return fail("status MSA_OK");
  if (strcmp(msa_status_string(MSA_ERR_DEVICE), "MSA_ERR_DEVICE") != 0) return fail("status");
  /* documents of 1, 64, 65 and 0 tokens in chunks of 64: 1 + 1 + 2 + 0 chunks */
  const int64_t off[5] = {0, 1, 65, 130, 130};
  if (msa_count_chunks(off, 4, 64) != 4) return fail("count_chunks");
  const int64_t bad[3] = {0, 5, 3};
  if (msa_count_chunks(bad, 2, 64) != -1) return fail("count_chunks order");
  /* k larger than the bank: refused on the host before any device work */
  const int64_t coff[3] = {0, 2, 4};
  int32_t ids[8];
  float sc[8];
  char ws[256];
  const msa_status s = msa_route_topk((const void*)ws, 1, 1, 8, (const void*)ws, NULL, NULL, coff,
                                      2, 4, 8, 128, MSA_BF16, 3, NULL, ids, sc, NULL, ws,
                                      sizeof ws, NULL);
  if (s != MSA_ERR_INVALID_ARG) return fail("route k > n_docs");
  if (strlen(msa_last_error()) == 0) return fail("last_error");
  printf("ok\n");
  return 0;
}
"""


def test_header_compiles_and_links_as_c(msa, tmp_path):
    """The boundary from plain C: msa.h compiles as C11 with -pedantic -Werror, the program links
    against libmsa.so, and host-side calls (version, status strings, the chunk count, a
    rejected routing call with its message) behave as documented, without a GPU."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "caller.c"
    src.write_text(C_CALLER)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(msa.LIB_PATH)
    libname = os.path.basename(msa.LIB_PATH)
    assert libname.startswith("lib") and libname.endswith(".so")
    subprocess.run([cc, "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-l" + libname[3:-3], "-Wl,-rpath," + libdir],
                   check=True, capture_output=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"
