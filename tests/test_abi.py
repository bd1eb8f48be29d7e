"""The C-ABI library on the CPU: it loads without a GPU, exports every function include/attn.h
declares, and rejects bad arguments before any CUDA call (no compute call is made here)."""
import ctypes
import os
import re
import subprocess

import pytest

from exact_attention_161_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def api():
    build.build()
    from exact_attention_161_b200 import api as api_mod
    return api_mod


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree(api):
    assert declared_functions() == sorted(api.SIGNATURES)


def test_library_exports_every_declared_symbol(api):
    lib = ctypes.CDLL(api.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_version_and_error_strings(api):
    assert "sm_100a" in api.version()
    assert api.last_error() == ""


FAKE = ctypes.c_void_p(0x10000)      # never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p(0x10008)


def _fwd(api, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, B=1, Hq=4, Hkv=2, N=128, D=128, causal=1, window=0,
         rope=0.0, scale=0.0):
    return api.lib.attn_fwd(q, k, v, o, lse, B, Hq, Hkv, N, D, causal, window, rope, scale, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), 1), (dict(o=None), 1), (dict(k=MISALIGNED), 1), (dict(lse=MISALIGNED), 1),
    (dict(B=0), 1), (dict(N=0), 1), (dict(Hq=3, Hkv=2), 1), (dict(causal=2), 1),
    (dict(causal=0, window=16), 1), (dict(scale=float("nan")), 1), (dict(rope=float("inf")), 1),
    (dict(D=96), 2), (dict(D=256), 2), (dict(B=65535, Hq=65535, Hkv=1), 2),
])
def test_fwd_validation(api, kw, expect):
    assert _fwd(api, **kw) == expect
    assert api.last_error() != ""


def _fwd_pos(api, causal=1, half=0, ps=1.0, ntk=1.0, alibi=None, rope=10000.0):
    return api.lib.attn_fwd_pos(FAKE, FAKE, FAKE, FAKE, None, 1, 4, 2, 128, 128, causal, 0, rope, half, ps, ntk, alibi,
                                0.0, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(half=2), 1), (dict(ps=0.0), 1), (dict(ps=float("inf")), 1), (dict(ntk=-1.0), 1),
    (dict(causal=0, alibi=FAKE), 1), (dict(alibi=ctypes.c_void_p(0x10002)), 1),
])
def test_fwd_pos_validation(api, kw, expect):
    assert _fwd_pos(api, **kw) == expect


def _fwd_fp8(api, D=128, dq=1.0, dk=1.0, dv=1.0, causal=1, window=0):
    return api.lib.attn_fwd_fp8(FAKE, FAKE, FAKE, FAKE, None, 1, 4, 2, 128, D, causal, window, dq, dk, dv, 0.0, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(dq=0.0), 1), (dict(dv=float("nan")), 1), (dict(dk=-1.0), 1), (dict(causal=0, window=8), 1),
    (dict(D=64), 2),
])
def test_fwd_fp8_validation(api, kw, expect):
    assert _fwd_fp8(api, **kw) == expect


def _dec(api, num_seqs=2, max_blocks=8, num_pages=16, page_size=16, Hq=8, Hkv=2, D=128, ws_bytes=None,
         ws=FAKE, q=FAKE, bt=FAKE):
    if ws_bytes is None:
        ws_bytes = api.decode_workspace_size(num_seqs, max_blocks, page_size, Hq, D)
    return api.lib.attn_decode_paged(q, FAKE, FAKE, bt, FAKE, num_seqs, max_blocks, num_pages, page_size, Hq, Hkv, D,
                                     0.0, FAKE, None, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), 1), (dict(ws=None), 1), (dict(bt=ctypes.c_void_p(0x10002)), 1), (dict(num_seqs=0), 1),
    (dict(Hq=6, Hkv=4), 1), (dict(ws_bytes=16), 1), (dict(page_size=32), 2), (dict(D=80), 2),
    (dict(Hq=32, Hkv=1), 2), (dict(num_seqs=70000), 2),
])
def test_decode_validation(api, kw, expect):
    assert _dec(api, **kw) == expect


def test_workspace_size(api):
    # per (sequence, head, 512-token split): D partial outputs plus (max, sum), fp32, 256-B rounded
    assert api.decode_workspace_size(64, 1024, 16, 32, 128) == 64 * 32 * 32 * 130 * 4
    assert api.decode_workspace_size(1, 1, 16, 1, 64) == 512
    assert api.decode_workspace_size(0, 1, 16, 1, 64) == 0


def _bwd(api, q=FAKE, lse=FAKE, dq=FAKE, ws=FAKE, B=1, Hq=4, Hkv=2, N=128, D=128, causal=1, window=0, rope=0.0,
         scale=0.0, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = api.bwd_workspace_size(B, Hq, Hkv, N, D, rope) if B > 0 and Hq > 0 and Hkv > 0 and N > 0 else 0
    return api.lib.attn_bwd(q, FAKE, FAKE, FAKE, lse, FAKE, dq, FAKE, FAKE, B, Hq, Hkv, N, D, causal, window, rope,
                            scale, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), 1), (dict(dq=None), 1), (dict(ws=None), 1), (dict(lse=ctypes.c_void_p(0x10002)), 1),
    (dict(dq=MISALIGNED), 1), (dict(N=0), 1), (dict(Hq=3, Hkv=2), 1), (dict(causal=0, window=8), 1),
    (dict(scale=float("inf")), 1), (dict(ws_bytes=256), 1), (dict(rope=10000.0, ws_bytes=70000), 1),
    (dict(D=96), 2), (dict(B=65535, Hq=65535, Hkv=1), 2),
])
def test_bwd_validation(api, kw, expect):
    assert _bwd(api, **kw) == expect
    assert api.last_error() != ""


def test_bwd_workspace_size(api):
    # fp32 (-LSE log2 e, -D_i) and fp32 dq sums per query row padded to 128-row tiles, each 256-B
    # rounded; with RoPE also the rotated Q and K in bf16, each 256-B rounded
    assert api.bwd_workspace_size(1, 4, 2, 128, 128) == 4 * 128 * 2 * 4 + 4 * 128 * 128 * 4
    assert api.bwd_workspace_size(1, 1, 1, 1, 64) == 1024 + 128 * 64 * 4
    assert api.bwd_workspace_size(2, 32, 8, 8192, 128, 10000.0) == (2 * 32 * 8192 * 2 * 4 + 2 * 32 * 8192 * 128 * 4
                                                                     + 2 * 32 * 8192 * 128 * 2
                                                                     + 2 * 8 * 8192 * 128 * 2)
    assert api.bwd_workspace_size(1, 2, 1, 3, 64, 10000.0) == 2 * 128 * 2 * 4 + 2 * 128 * 64 * 4 + 768 + 512
    assert api.bwd_workspace_size(0, 4, 2, 128, 128) == 0


def test_decode_noalloc_limit_is_checked_before_any_launch(api):
    """2048 sequences x 32 heads x 32 splits x (128 + 2) floats exceed the fixed 40 MiB array: the
    call is rejected on the host, naming the limit; smaller requests pass that check."""
    st = api.lib.attn_decode_paged_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, 2048, 1024, 100, 16, 32, 8, 128, 0.0, FAKE,
                                           None, None)
    assert st == api.ATTN_ERR_INVALID_ARG and "no-alloc limit" in api.last_error()
    assert api.decode_workspace_size(2048, 1024, 16, 32, 128) > 40 << 20
    assert api.decode_workspace_size(64, 1024, 16, 32, 128) <= 40 << 20


def _step(api, q_len=2, Hq=8, Hkv=2, D=128, k_new=FAKE, v_new=FAKE, ws_bytes=None, rope=0.0):
    if ws_bytes is None:
        ws_bytes = api.decode_step_workspace_size(2, q_len, 8, 16, Hq, D)
    return api.lib.attn_decode_step(FAKE, k_new, v_new, FAKE, FAKE, FAKE, FAKE, 2, q_len, 8, 16, 16, Hq, Hkv, D,
                                    rope, 0.0, FAKE, None, FAKE, ws_bytes, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q_len=0), 1), (dict(k_new=None), 1), (dict(v_new=MISALIGNED), 1), (dict(ws_bytes=16), 1),
    (dict(rope=float("nan")), 1), (dict(q_len=65), 2), (dict(D=96), 2), (dict(Hq=34, Hkv=2), 2),
])
def test_decode_step_validation(api, kw, expect):
    assert _step(api, **kw) == expect


def test_decode_step_workspace_size(api):
    # the split's partial states per (sequence, new token, head, chunk), then the rotated queries
    assert api.decode_step_workspace_size(64, 4, 1024, 16, 32, 128) == 64 * 4 * 32 * 32 * 130 * 4 + 64 * 4 * 32 * 128 * 2
    assert api.decode_step_workspace_size(64, 1, 1024, 16, 32, 128) == (
        api.decode_workspace_size(64, 1024, 16, 32, 128) + 64 * 32 * 128 * 2)
    assert api.decode_step_workspace_size(1, 0, 1, 16, 1, 64) == 0


def test_device_status_needs_out_pointer(api):
    assert api.lib.attn_get_device_status(None, None) == 1


def test_header_is_plain_c_and_a_c_program_links(api, tmp_path):
    """include/attn.h compiles as strict C99 on its own (no CUDA or C++ header needed), and a C
    program built against it links with the library, finds every declared function and gets the
    documented answers from the calls that need no GPU: the version string, a null-pointer
    rejection with its message, and the workspace sizes the Python binding also reports."""
    table = ",\n    ".join("(fn)%s" % f for f in declared_functions())
    src = tmp_path / "use_attn.c"
    src.write_text("""#include "attn.h"
#include <stdio.h>
#include <string.h>
typedef void (*fn)(void);
static const fn every_entry_point[] = {
    %s
};
int main(void) {
    size_t i;
    for (i = 0; i < sizeof every_entry_point / sizeof every_entry_point[0]; ++i)
        if (!every_entry_point[i]) return 10;
    if (!strstr(attn_version(), "sm_100a")) return 11;
    if (attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 1, 1, 128, 64, 1, 0, 0.f, 0.f, NULL) != ATTN_ERR_INVALID_ARG)
        return 12;
    if (attn_last_error()[0] == 0) return 13;
    printf("%%zu %%zu %%zu\\n", attn_bwd_workspace_size(2, 32, 8, 8192, 128, 5e5f),
           attn_decode_workspace_size(64, 1024, 16, 32, 128),
           attn_decode_step_workspace_size(64, 4, 1024, 16, 32, 128));
    return 0;
}
""" % table)
    exe = tmp_path / "use_attn"
    lib_dir = os.path.dirname(api.LIB_PATH)
    lib_name = os.path.basename(api.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                    os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", lib_dir,
                    "-l:" + lib_name, "-Wl,-rpath," + lib_dir], check=True)
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0, (run.returncode, run.stderr)
    sizes = [int(x) for x in run.stdout.split()]
    assert sizes == [api.bwd_workspace_size(2, 32, 8, 8192, 128, 5e5),
                     api.decode_workspace_size(64, 1024, 16, 32, 128),
                     api.decode_step_workspace_size(64, 4, 1024, 16, 32, 128)]
