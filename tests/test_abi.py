"""The C ABI without a GPU: the library loads, exports every entry point include/fa.h
declares, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

from exact_attention_126_b200 import build, fa

HEADER = os.path.join(build.INCLUDE, "fa.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return fa.library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    assert set(names) == set(fa.EXPORTED), names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_only_the_declared_entry_points_are_exported(lib):
    import shutil
    import subprocess
    nm = shutil.which("nm")
    if nm is None:
        pytest.skip("nm is not available")
    out = subprocess.run([nm, "-D", "--defined-only", fa.LIBRARY], capture_output=True,
                         text=True, check=True).stdout
    names = {line.split()[-1] for line in out.splitlines() if line.strip()}
    names = {n for n in names if not n.startswith(("_init", "_fini"))}
    assert names == set(declared_functions()), sorted(names ^ set(declared_functions()))


def test_status_strings(lib):
    for code, name in fa.STATUS_NAMES.items():
        assert fa.fa_status_string(code).startswith(name)
    assert fa.fa_status_string(99) == "FA_ERR_UNKNOWN"


W = fa.fa_window_t
A = 0x10000  # a fake, 16-byte aligned "device" address: never dereferenced on these paths


def fwd(lib, q=A, k=A, v=A, o=A, lse=A, B=1, H=1, N=128, d=64, scale=0.125, causal=0,
        window=(-1, -1)):
    return lib.fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, W(*window), None)


def test_fwd_rejects_bad_arguments(lib):
    assert fwd(lib, q=None) == 1
    assert fwd(lib, lse=None) == 1
    assert fwd(lib, q=A + 8) == 3
    assert fwd(lib, o=A + 2) == 3
    assert fwd(lib, d=96) == 2
    assert fwd(lib, d=32) == 2
    assert fwd(lib, B=-1) == 1
    assert fwd(lib, N=-5) == 1
    assert fwd(lib, scale=0.0) == 1
    assert fwd(lib, scale=-0.1) == 1
    assert fwd(lib, scale=float("nan")) == 1
    assert fwd(lib, scale=float("inf")) == 1
    assert fwd(lib, window=(-2, -1)) == 1
    assert fwd(lib, window=(5, -3)) == 1
    assert fwd(lib, B=1 << 12, H=1 << 12, N=256, d=64) == 2  # >= 2^31 elements
    # more than 65535 (batch, head) pairs is accepted (no grid dimension is limited by it)
    assert lib.fa_bwd_workspace_bytes(1 << 17, 1, 64, 128) == 2 * (1 << 17) * 128 * 4


def test_empty_problem_is_a_no_op(lib):
    # nothing is launched, so even null pointers are accepted
    assert fwd(lib, q=None, k=None, v=None, o=None, lse=None, N=0) == 0
    assert fwd(lib, B=0) == 0
    assert fwd(lib, H=0) == 0
    assert lib.fa_bwd_workspace_bytes(1, 1, 0, 64) == 0


def test_workspace_size(lib):
    # two fp32 arrays (LSE*log2e and delta) of B*H rows padded to whole 128-row tiles
    assert lib.fa_bwd_workspace_bytes(2, 8, 4096, 64) == 2 * 2 * 8 * 4096 * 4
    assert lib.fa_bwd_workspace_bytes(1, 1, 3, 64) == 2 * 128 * 4
    assert lib.fa_bwd_workspace_bytes(1, 2, 129, 128) == 2 * 2 * 256 * 4
    assert lib.fa_bwd_workspace_bytes(1, 1, 3, 80) == 0


def bwd(lib, ws=A, ws_bytes=1 << 20, **kw):
    args = dict(q=A, k=A, v=A, o=A, do=A, lse=A, dq=A, dk=A, dv=A, B=1, H=1, N=128, d=64,
                scale=0.125, causal=0, window=(-1, -1))
    args.update(kw)
    a = args
    return lib.fa_bwd(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"], a["dk"],
                      a["dv"], a["B"], a["H"], a["N"], a["d"], a["scale"], a["causal"],
                      W(*a["window"]), ws, ws_bytes, None)


def test_bwd_rejects_bad_arguments(lib):
    assert bwd(lib, dq=None) == 1
    assert bwd(lib, ws=None) == 1
    assert bwd(lib, dv=A + 4) == 3
    assert bwd(lib, ws_bytes=2 * 128 * 4 - 1) == 4
    assert bwd(lib, d=256) == 2
    assert bwd(lib, window=(-7, 0)) == 1
    assert lib.fa_bwd_preprocess(A, None, A, A, 1, 1, 128, 64, None, None) == 1
    assert lib.fa_bwd_preprocess(A, A, A, A + 8, 1, 1, 128, 64, None, None) == 3
    assert lib.fa_bwd_dkdv(A, A, A, A, A, A, A + 1, 1, 1, 128, 64, 0.1, 0, W(-1, -1),
                           None, None) == 3
    assert lib.fa_bwd_dq(A, A, A, A, A, A, 1, 1, 128, 128, -1.0, 0, W(-1, -1), None,
                         None) == 1


def test_options_are_checked(lib):
    def fwd_ex(opt, q=A, d=64):
        return lib.fa_fwd_ex(q, A, A, A, A, 1, 2, 128, d, 0.125, 0, W(-1, -1), opt, None)

    def bwd_ex(opt, ws_bytes=1 << 20):
        return lib.fa_bwd_ex(A, A, A, A, A, A, A, A, A, 1, 2, 128, 64, 0.125, 0, W(-1, -1), opt,
                             A, ws_bytes, None)

    def O(**kw):
        return fa.fa_options_t(**kw)

    assert fwd_ex(O(alibi_slopes=A + 2)) == 3       # slopes not 4-byte aligned
    assert fwd_ex(O(o_low=A + 8)) == 3              # o_low not 16-byte aligned
    assert fwd_ex(O(dropout_p=1.0)) == 1            # dropout probability >= 1
    assert fwd_ex(O(dropout_p=-0.1)) == 1           # negative probability
    assert fwd_ex(O(dropout_p=0.999)) == 1          # rounds to 256/256: nothing kept
    assert fwd_ex(O(dropout_p=float("nan"))) == 1
    assert fwd_ex(O(dropout_p=0.1, dropout_offset=1 << 32)) == 1  # offset wider than 32 bits
    assert fwd_ex(O(flags=2)) == 1                  # unknown flag
    assert fwd_ex(O(seq_lengths=A + 2)) == 3        # lengths not 4-byte aligned
    assert fwd_ex(O(key_padding=A + 1), q=None) == 1
    assert fwd_ex(None, d=96) == 2
    assert bwd_ex(O(o_low=A + 4)) == 3
    assert bwd_ex(O(dropout_p=1.5)) == 1
    assert bwd_ex(None, ws_bytes=8) == 4
    # the fused backward (head_dim 64) needs the dQ accumulator as well
    stats = 2 * 2 * 128 * 4
    assert bwd_ex(O(flags=1), ws_bytes=stats) == 4
    assert lib.fa_bwd_workspace_bytes_ex(1, 2, 128, 64, ctypes.byref(O(flags=1))) == \
        stats + 2 * 128 * 64 * 4
    assert lib.fa_bwd_workspace_bytes_ex(1, 2, 128, 64, None) == stats
    assert lib.fa_bwd_workspace_bytes_ex(1, 2, 128, 128, ctypes.byref(O(flags=1))) == stats
    assert lib.fa_bwd_workspace_bytes_ex(1, 2, 128, 64, ctypes.byref(O(flags=4))) == 0
    # a variable-length batch adds, last, the tables of its schedule: start (T + 1 ints),
    # the batch entries by length (B ints) and T + 1 ints of scratch, rounded to 256 bytes
    def sched(B, T):
        return (4 * (2 * (T + 1) + B) + 255) // 256 * 256
    for B, H, N, d, flags in ((1, 2, 128, 64, 0), (3, 2, 1000, 128, 0), (70, 1, 4096, 64, 1)):
        base = lib.fa_bwd_workspace_bytes_ex(B, H, N, d, ctypes.byref(O(flags=flags)))
        got = lib.fa_bwd_workspace_bytes_ex(B, H, N, d,
                                            ctypes.byref(O(flags=flags, seq_lengths=A)))
        assert got == base + sched(B, (N + 127) // 128)
    assert bwd_ex(O(seq_lengths=A), ws_bytes=stats) == 4
    # a packed batch: cumulative lengths 4-byte aligned, exclusive with seq_lengths, a token
    # count >= 0, not with the fused backward; no tokens is an empty call
    assert fwd_ex(O(cu_seqlens=A + 2, total_tokens=5)) == 3
    assert fwd_ex(O(cu_seqlens=A, seq_lengths=A, total_tokens=5)) == 1
    assert fwd_ex(O(cu_seqlens=A, total_tokens=-1)) == 1
    assert bwd_ex(O(cu_seqlens=A, total_tokens=5, flags=1)) == 2
    assert lib.fa_fwd_ex(None, None, None, None, None, 1, 2, 128, 64, 0.125, 0, W(-1, -1),
                         O(cu_seqlens=A, total_tokens=0), None) == 0
    assert lib.fa_fwd_ex(A, A, A, A, A, 1, 2, 128, 64, 0.125, 0, W(-1, -1),
                         O(cu_seqlens=A, total_tokens=1 << 24), None) == 2  # >= 2^31 elements
    assert lib.fa_bwd_workspace_bytes_ex(3, 2, 1000, 128,
                                         ctypes.byref(O(cu_seqlens=A, total_tokens=9))) == \
        lib.fa_bwd_workspace_bytes_ex(3, 2, 1000, 128, None) + sched(3, 8)
    assert lib.fa_bwd_fused(A, A, A, A, A, A, A, 1, 1, 128, 128, 0.1, 0, W(-1, -1), None,
                            None) == 2   # the fused pass is for head_dim 64
    assert lib.fa_bwd_dq_convert(A, None, 1, 1, 128, 64, 0.1, None) == 1
    assert lib.fa_bwd_dq_convert(A, A, 1, 1, 128, 128, 0.1, None) == 2
    # empty problems launch nothing, whatever the options
    assert lib.fa_fwd_ex(None, None, None, None, None, 1, 2, 0, 64, 0.125, 0, W(-1, -1),
                         O(alibi_slopes=A + 2, dropout_p=0.5), None) == 0


def test_fp8_forward_rejects_bad_arguments(lib):
    def fwd8(q=A, d=128, qs=1.0, ks=1.0, vs=1.0, scale=0.09, o=A):
        return lib.fa_fwd_fp8(q, A, A, qs, ks, vs, o, A, 1, 2, 128, d, scale, 1, W(-1, -1), None)

    assert fwd8(d=64) == 2            # the e4m3 forward is for head_dim 128
    assert fwd8(qs=0.0) == 1
    assert fwd8(ks=float("nan")) == 1
    assert fwd8(vs=-1.0) == 1
    assert fwd8(scale=0.0) == 1
    assert fwd8(q=None) == 1
    assert fwd8(o=A + 2) == 3
    assert lib.fa_fwd_fp8(None, None, None, 1.0, 1.0, 1.0, None, None, 0, 2, 128, 128, 0.1, 0,
                          W(-1, -1), None) == 0


def test_options_struct_layout(tmp_path):
    """The binding's fa_options_t has the C header's layout (checked against the header
    compiled by the host C compiler)."""
    import ctypes
    import shutil
    import subprocess
    O = fa.fa_options_t
    names = ["alibi_slopes", "key_padding", "o_low", "dropout_p", "flags", "dropout_seed",
             "dropout_offset", "seq_lengths", "cu_seqlens", "total_tokens"]
    py = [ctypes.sizeof(O)] + [getattr(O, n).offset for n in names]
    assert py == [72, 0, 8, 16, 24, 28, 32, 40, 48, 56, 64]
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    src = tmp_path / "layout.c"
    src.write_text('#include <stddef.h>\n#include <stdio.h>\n#include "fa.h"\nint main(void) {\n'
                   '  printf("%zu", sizeof(fa_options_t));\n' +
                   "".join('  printf(" %%zu", offsetof(fa_options_t, %s));\n' % n for n in names) +
                   "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", build.INCLUDE, str(src), "-o", str(exe)],
                   check=True)
    c = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True,
                                        check=True).stdout.split()]
    assert c == py


def test_python_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(fa, "_LIB", None)
    monkeypatch.setattr(fa, "LIBRARY", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        fa.library()


def test_alibi_rejects_bad_arguments(lib):
    def fwd_alibi(slopes=A, q=A, d=64, scale=0.125):
        return lib.fa_fwd_alibi(q, A, A, A, A, 1, 2, 128, d, scale, 0, W(-1, -1), slopes, None)

    def bwd_alibi(slopes=A, ws_bytes=1 << 20, dk=A):
        return lib.fa_bwd_alibi(A, A, A, A, A, A, A, dk, A, 1, 2, 128, 64, 0.125, 0, W(-1, -1),
                                slopes, A, ws_bytes, None)

    assert fwd_alibi(slopes=None) == 1
    assert fwd_alibi(slopes=A + 2) == 3
    assert fwd_alibi(q=None) == 1
    assert fwd_alibi(d=80) == 2
    assert fwd_alibi(scale=0.0) == 1
    assert bwd_alibi(slopes=None) == 1
    assert bwd_alibi(slopes=A + 1) == 3
    assert bwd_alibi(dk=None) == 1
    assert bwd_alibi(ws_bytes=16) == 4
    # an empty problem launches nothing, with or without slopes
    assert lib.fa_fwd_alibi(None, None, None, None, None, 1, 2, 0, 64, 0.125, 0, W(-1, -1), None,
                            None) == 0
