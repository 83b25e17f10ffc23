"""The C ABI library loads without a GPU, exports every entry point its header declares, and
rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

from post_weight_quantization_12_b200 import _lib

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "gptq.h")
FAKE = ctypes.c_void_p(0x10000)   # never dereferenced: every call below fails validation first


def declared_functions():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    return sorted(set(re.findall(r"\b(gptq_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_path():
    names = declared_functions()
    for n in ("gptq_hessian_accumulate", "gptq_prepare_hinv", "gptq_quantize_layer",
              "gptq_workspace_size", "gptq_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(built_lib):
    lib = ctypes.CDLL(built_lib)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(_lib.SIGNATURES)


def test_status_strings_and_info_mapping(built_lib):
    assert _lib.status_string(0) == "GPTQ_OK"
    assert "EINVAL" in _lib.status_string(1)
    assert _lib.info_status(0) == _lib.GPTQ_OK
    assert _lib.info_status(7) == _lib.GPTQ_ENOTPD
    assert _lib.info_status(-1) == _lib.GPTQ_ETIMEOUT
    assert _lib.load().gptq_version().decode().count(".") == 2


def test_workspace_sizes(built_lib):
    q = _lib.workspace_size(_lib.GPTQ_WS_QUANTIZE, 4096, 4096, 128)
    assert q >= 4096 * 128 * 4 and q % 256 == 0
    p = _lib.workspace_size(_lib.GPTQ_WS_PREPARE, 0, 4096, 0)
    assert p >= 4096 * 4096 * 4
    assert _lib.workspace_size(_lib.GPTQ_WS_QUANTIZE, 10, 10, 48) == 0
    assert _lib.workspace_size(99, 10, 10, 32) == 0


@pytest.mark.parametrize("bits,group,block,cols,ldw", [
    (1, -1, 128, 256, 256),      # bits below range
    (9, -1, 128, 256, 256),      # bits above range
    (4, 48, 32, 480, 480),       # group and block do not nest
    (4, 128, 128, 200, 200),     # cols not a multiple of the group
    (4, -1, 96, 256, 256),       # unsupported block
    (4, 0, 128, 256, 256),       # group 0
    (4, -1, 128, 256, 100),      # ldw < cols
])
def test_quantize_rejects_bad_arguments(built_lib, bits, group, block, cols, ldw):
    lib = _lib.load()
    st = lib.gptq_quantize_layer(FAKE, _lib.GPTQ_BF16, 64, cols, ldw, FAKE, bits, group, block,
                                 FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, FAKE, None)
    assert st == _lib.GPTQ_EINVAL


def test_other_entry_points_reject_bad_arguments(built_lib):
    lib = _lib.load()
    assert lib.gptq_hessian_accumulate(None, 128, FAKE, 0, 10, 128, FAKE, None) == _lib.GPTQ_EINVAL
    assert lib.gptq_hessian_accumulate(FAKE, 128, FAKE, 0, 10, 64, FAKE, None) == _lib.GPTQ_EINVAL
    # bf16 path needs 16-byte rows and base
    assert lib.gptq_hessian_accumulate(FAKE, 12, FAKE, 0, 10, 12, FAKE, None) == _lib.GPTQ_EINVAL
    assert lib.gptq_hessian_accumulate(FAKE, 128, FAKE, 0, 0, 128, FAKE, None) == _lib.GPTQ_OK
    assert lib.gptq_prepare_hinv(FAKE, FAKE, 128, 0, 0.01, FAKE, 1 << 30, FAKE, None) == \
        _lib.GPTQ_EINVAL
    assert lib.gptq_prepare_hinv(FAKE, FAKE, 128, 10, -1.0, FAKE, 1 << 30, FAKE, None) == \
        _lib.GPTQ_EINVAL
    assert lib.gptq_prepare_hinv(FAKE, FAKE, 128, 10, 0.01, FAKE, 16, FAKE, None) == \
        _lib.GPTQ_EWORKSPACE
    for route in (-1, 3):
        assert lib.gptq_prepare_hinv_route(FAKE, FAKE, 128, 10, 0.01, route, FAKE, 1 << 30, FAKE,
                                           None) == _lib.GPTQ_EINVAL
    assert lib.gptq_prepare_hinv_route(FAKE, FAKE, 128, 10, 0.01, _lib.GPTQ_ROUTE_REVERSED, FAKE,
                                       16, FAKE, None) == _lib.GPTQ_EWORKSPACE
    st = lib.gptq_quantize_layer(FAKE, _lib.GPTQ_FP32, 64, 128, 128, FAKE, 4, -1, 32, FAKE, FAKE,
                                 FAKE, FAKE, None, FAKE, 16, FAKE, None)
    assert st == _lib.GPTQ_EWORKSPACE
    assert lib.gptq_selftest_wait_timeout(FAKE, 0, None) == _lib.GPTQ_EINVAL
    assert lib.gptq_selftest_flag_timeout(None, FAKE, 50, None) == _lib.GPTQ_EINVAL
    assert lib.gptq_selftest_flag_timeout(FAKE, None, 50, None) == _lib.GPTQ_EINVAL
    assert lib.gptq_selftest_flag_timeout(FAKE, FAKE, 0, None) == _lib.GPTQ_EINVAL
    assert lib.gptq_selftest_flag_timeout(ctypes.c_void_p(0x10002), FAKE, 50, None) == \
        _lib.GPTQ_EINVAL


def test_w4a16_entry_points_reject_bad_arguments(built_lib):
    lib = _lib.load()
    BF, F32 = _lib.GPTQ_BF16, _lib.GPTQ_FP32
    pack = lib.gptq_pack_codes_4bit
    assert pack(None, 4, 64, 64, FAKE, None, None) == _lib.GPTQ_EINVAL
    assert pack(None, 0, 64, 64, None, None, None) == _lib.GPTQ_OK          # empty, no buffers
    assert pack(FAKE, 4, 60, 64, FAKE, None, None) == _lib.GPTQ_EINVAL      # cols % 8
    assert pack(FAKE, 4, 64, 60, FAKE, None, None) == _lib.GPTQ_EINVAL      # ldc < cols
    assert pack(FAKE, 4, 64, 68, FAKE, None, None) == _lib.GPTQ_EINVAL      # ldc % 8
    assert pack(FAKE, 0, 64, 64, FAKE, None, None) == _lib.GPTQ_OK          # empty: no-op
    pack3 = lib.gptq_pack_codes_3bit
    assert pack3(None, 4, 64, 64, FAKE, None, None) == _lib.GPTQ_EINVAL
    assert pack3(None, 0, 64, 64, None, None, None) == _lib.GPTQ_OK         # empty, no buffers
    assert pack3(FAKE, 4, 48, 64, FAKE, None, None) == _lib.GPTQ_EINVAL     # cols % 32
    assert pack3(FAKE, 4, 64, 60, FAKE, None, None) == _lib.GPTQ_EINVAL     # ldc < cols
    assert pack3(FAKE, 4, 64, 68, FAKE, None, None) == _lib.GPTQ_EINVAL     # ldc % 8
    mm = lib.gptq_w4a16_matmul

    def call(rows=64, cols=256, group=128, dtype=BF, n=1, ldx=256, ldy=64, x=FAKE):
        return mm(FAKE, FAKE, FAKE, rows, cols, group, x, dtype, n, ldx, FAKE, ldy, None, None)

    assert call(x=None) == _lib.GPTQ_EINVAL
    assert call(cols=240, group=-1, ldx=240) == _lib.GPTQ_EINVAL        # cols % 32
    assert call(group=64) == _lib.GPTQ_EINVAL                            # group not a 128 multiple
    assert call(cols=384, group=256, ldx=384) == _lib.GPTQ_EINVAL        # group does not divide
    assert call(group=0) == _lib.GPTQ_EINVAL
    assert call(ldx=200) == _lib.GPTQ_EINVAL                             # ldx < cols
    assert call(ldx=260) == _lib.GPTQ_EINVAL                             # ldx % 8
    assert call(ldy=10) == _lib.GPTQ_EINVAL                              # ldy < rows
    assert call(n=-1) == _lib.GPTQ_EINVAL
    assert call(dtype=F32) == _lib.GPTQ_EUNSUPPORTED
    assert call(n=65535 * 128 + 1) == _lib.GPTQ_EUNSUPPORTED          # past the product's grid
    assert call(cols=(1 << 22) + 128, ldx=(1 << 22) + 128) == _lib.GPTQ_EUNSUPPORTED
    assert call(rows=0) == _lib.GPTQ_OK and call(n=0) == _lib.GPTQ_OK    # empty: no-op
    assert call(n=0, x=None) == _lib.GPTQ_OK
    assert _lib.info_status(_lib.GPTQ_INFO_BAD_CODE) == _lib.GPTQ_EINVAL


def test_rotation_entry_points(built_lib):
    lib = _lib.load()
    for n, b in ((4096, 4096), (11008, 256), (12288, 4096), (49152, 4096), (96, 32), (0, 0)):
        assert _lib.hadamard_block(n) == b
    BF, F32 = _lib.GPTQ_BF16, _lib.GPTQ_FP32
    rot = lib.gptq_hadamard_rotate

    def call(rows=4, n=256, ldx=256, xd=BF, yd=BF, ldy=256, x=FAKE, y=ctypes.c_void_p(0x20000)):
        return rot(x, xd, rows, n, ldx, None, y, yd, ldy, None)

    assert call(n=240, ldx=240, ldy=240) == _lib.GPTQ_EINVAL         # n % 32
    assert call(ldx=200) == _lib.GPTQ_EINVAL                         # ldx < n
    assert call(ldx=260) == _lib.GPTQ_EINVAL                         # ldx * 2 % 16
    assert call(xd=F32, ldx=258) == _lib.GPTQ_EINVAL                 # ldx * 4 % 16
    assert call(yd=7) == _lib.GPTQ_EINVAL
    assert call(x=None) == _lib.GPTQ_EINVAL
    assert call(y=FAKE, yd=F32) == _lib.GPTQ_EINVAL                  # in place, dtype differs
    assert call(rows=0, x=None, y=None) == _lib.GPTQ_OK              # empty: no-op


def test_obq_entry_point_rejects_bad_arguments(built_lib):
    lib = _lib.load()

    def call(rows=4, cols=64, ldw=64, bits=4, mode=1, w=FAKE):
        return lib.gptq_obq_quantize(w, rows, cols, ldw, FAKE, bits, mode, FAKE, FAKE, None, None,
                                     None, None, None)

    assert call(cols=0) == _lib.GPTQ_EINVAL
    assert call(ldw=32) == _lib.GPTQ_EINVAL
    assert call(bits=1) == _lib.GPTQ_EINVAL and call(bits=9) == _lib.GPTQ_EINVAL
    assert call(mode=2) == _lib.GPTQ_EINVAL
    assert call(w=None) == _lib.GPTQ_EINVAL
    assert call(cols=129, ldw=129) == _lib.GPTQ_EUNSUPPORTED
    assert call(rows=0, w=None) == _lib.GPTQ_OK



def test_header_compiles_as_c_and_links(built_lib, tmp_path):
    """include/gptq.h is plain C (C99, pedantic) and a C program links against the library."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_gptq.c"
    src.write_text('#include "gptq.h"\n#include <stdio.h>\n'
                   'int main(void) { printf("%s %d\\n", gptq_version(), '
                   'gptq_hadamard_block(11008)); return 0; }\n')
    exe = tmp_path / "use_gptq"
    inc = os.path.join(os.path.dirname(HEADER))
    libdir = os.path.dirname(built_lib)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", inc,
                    str(src), "-o", str(exe), "-L", libdir, "-l:libgptq_b200.so",
                    "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert out[0].count(".") == 2 and out[1] == "256"
