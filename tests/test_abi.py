"""CPU checks of the C-ABI library: it loads, exports every declared symbol,
and rejects host-detectable bad arguments without touching the device."""

import ctypes
import os
import re

import pytest

from mla_latent_kv_35_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "mla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from mla_latent_kv_35_b200 import build
    build.build()
    return B.lib()


def test_header_and_binding_agree():
    assert _declared() == sorted(B.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(B.LIB_PATH)
    for name in _declared():
        assert hasattr(raw, name), name


def test_status_strings(lib):
    for code in range(6):
        assert B.mla_status_string(code)
    assert B.mla_status_string(99) == "unknown status"


def _dims(**over):
    d = dict(n_heads=128, d_nope=128, d_latent=512, d_rope=64, d_v=128, d_model=5120,
             page_size=64, scale=192 ** -0.5, rope_base=10000.0, dtype="bf16")
    d.update(over)
    return B.MLADims(**d)


def test_bad_arguments_rejected_on_host(lib):
    d = ctypes.byref(_dims().c())
    NULL = None
    # null buffers
    assert lib.mla_project(d, NULL, NULL, NULL, 4, 5120, 256, NULL) == 1
    assert lib.mla_decode(d, NULL, NULL, 10, NULL, 4, NULL, 2, 1, 0, NULL, 0, NULL, NULL,
                          NULL) == 1
    # S_q out of range
    assert lib.mla_decode(d, NULL, NULL, 10, NULL, 4, NULL, 2, 3, 0, NULL, 0, NULL, NULL,
                          NULL) == 1
    # odd RoPE width
    bad = ctypes.byref(_dims(d_rope=63).c())
    assert lib.mla_rope(bad, NULL, 0, 0, 1, NULL, 0, 0, NULL, 4, NULL) == 1
    # empty work is a no-op, even with null pointers
    assert lib.mla_project(d, NULL, NULL, NULL, 0, 5120, 256, NULL) == 0
    assert lib.mla_cache_append(d, NULL, 0, NULL, 0, NULL, NULL, NULL, 4, NULL, 8, 0, NULL) == 0
    assert lib.mla_decode(d, NULL, NULL, 10, NULL, 4, NULL, 0, 1, 0, NULL, 0, NULL, NULL,
                          NULL) == 0


def test_workspace_sizes_grow_with_work(lib):
    d = _dims()
    a = B.mla_decode_workspace_size(d, 16, 1, 74)
    b = B.mla_decode_workspace_size(d, 128, 1, 74)
    c = B.mla_decode_workspace_size(d, 128, 2, 74)
    assert 0 < a < b < c
    assert B.mla_out_proj_scratch_size(d, 128) >= 128 * 128 * (512 + 128) * 2
    f32 = _dims(dtype="f32", n_heads=8, d_nope=32, d_latent=64, d_rope=16, d_v=32,
                d_model=256)
    assert B.mla_out_proj_scratch_size(f32, 2) >= 2 * 8 * 32 * 4


def test_header_is_plain_c_and_a_c_program_links(tmp_path, lib):
    """include/mla.h compiles as pedantic C99 and a C program links against
    libmla_b200.so and calls it (host-only calls: no GPU needed)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "probe.c"
    src.write_text(
        "#include <stdio.h>\n#include \"mla.h\"\n"
        "int main(void) {\n"
        "  mla_dims d = {128, 128, 512, 64, 128, 5120, 64, 0.0721687836f, 10000.0f, MLA_BF16};\n"
        "  printf(\"%s|%zu\\n\", mla_status_string(MLA_ERR_BOUNDS),\n"
        "         mla_decode_workspace_size(&d, 128, 1, 74));\n"
        "  return 0;\n}\n")
    libdir = os.path.dirname(B.LIB_PATH)
    exe = tmp_path / "probe"
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                        "-I", os.path.join(ROOT, "include"), str(src), "-L", libdir,
                        "-lmla_b200", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True,
                         check=True).stdout.strip().split("|")
    assert out[0] == B.mla_status_string(5)
    assert int(out[1]) == B.mla_decode_workspace_size(_dims(), 128, 1, 74)
