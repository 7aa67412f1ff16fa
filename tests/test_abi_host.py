"""Host-side checks of the C ABI (no GPU): the library loads, exports every
function include/flarepp.h declares, and rejects bad arguments before any
device work."""
import ctypes
import subprocess

import pytest

import rank_latent_attention_b200 as flare

BF16, F32 = 1, 0


@pytest.fixture(scope="module")
def L():
    return flare.lib()


def test_header_declares_the_mixer_calls():
    names = flare.header_functions()
    for n in ("flare_encode", "flare_decode", "flarepp_mix"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", flare.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in flare.header_functions() if n not in exported]
    assert not missing, missing
    for n in flare.header_functions():
        getattr(L, n)  # resolvable through ctypes as well


def test_status_strings(L):
    assert L.flare_status_string(0) == b"ok"
    assert L.flare_status_string(4) == b"kernel wait timed out"
    assert L.flare_status_string(99) == b"unknown status"


@pytest.mark.parametrize("B,H,N,M,D,dtype,expect", [
    (1, 1, 10, 16, 64, BF16, 1),     # valid sizes, null pointers -> invalid argument
    (0, 1, 10, 16, 64, BF16, 1),     # B < 1
    (1, 1, 0, 16, 64, BF16, 1),      # N < 1
    (1, 1, 10, 17, 64, BF16, 2),     # M not a multiple of 16 on bf16
    (1, 1, 10, 272, 64, BF16, 2),    # M > 256
    (1, 1, 10, 16, 48, BF16, 2),     # D not in {16,32,64,128}
    (1, 1, 10, 16, 64, 7, 1),        # unknown dtype
    (300, 300, 10, 16, 64, BF16, 2), # B*H > 65535
    (1, 1, 1 << 31, 16, 64, BF16, 2),  # N too large
])
def test_mix_rejects_before_launch(L, B, H, N, M, D, dtype, expect):
    rc = L.flarepp_mix(None, None, None, None, B, H, N, M, D, dtype, None, 0, None)
    assert rc == expect


def test_f32_accepts_any_m(L):
    # M = 17 is fine on the fp32 path; null pointers are then the only problem
    assert L.flarepp_mix(None, None, None, None, 1, 1, 10, 17, 16, F32, None, 0, None) == 1


def test_host_pointer_is_rejected(L):
    buf = (ctypes.c_uint8 * 4096)()
    p = ctypes.cast(buf, ctypes.c_void_p)
    assert L.flare_decode(p, p, 0, p, p, 1, 1, 8, 16, 16, BF16, None) == 1
    assert L.flare_encode(p, 2, p, p, p, 1, 1, 8, 16, 16, BF16, None, 0, None) == 1  # bad q_batched


def test_workspace_sizes(L):
    assert L.flarepp_workspace_size(1, 1, 10, 17, 64, BF16) == 0
    a = L.flarepp_workspace_size(1, 16, 1 << 20, 256, 64, BF16)
    b = L.flare_encode_workspace_size(1, 16, 1 << 20, 256, 64, BF16)
    assert a > b > 0 and a % 256 == 0
    # the mix workspace holds the encode partials plus Q_dyn and Z (bf16)
    assert a - b >= 2 * 16 * 256 * 64 * 2


def test_backward_and_shard_sizes(L):
    # saved state: Q_dyn and Z (dtype) then two fp32 log-sum-exps, each region 256-byte aligned
    def r(x):
        return (x + 255) // 256 * 256
    BH, M, D = 16, 256, 64
    assert L.flarepp_saved_bytes(1, 16, M, D, BF16) == 2 * r(BH * M * D * 2) + 2 * r(BH * M * 4)
    assert L.flarepp_saved_bytes(1, 16, M, D, F32) == 2 * r(BH * M * D * 4) + 2 * r(BH * M * 4)
    assert L.flarepp_saved_bytes(1, 1, 17, 64, BF16) == 0          # bf16 needs M % 16 == 0
    assert L.flarepp_saved_bytes(1, 1, 16, 64, 2) == 0             # fp32-output mode has no backward
    wb = L.flarepp_mix_backward_workspace_size(1, 16, 1 << 20, M, D, BF16)
    # it holds the encode workspace, the per-token statistics (8 bytes a token) and more
    assert wb % 256 == 0 and wb > L.flare_encode_workspace_size(1, 16, 1 << 20, M, D, BF16) + 8 * BH * (1 << 20)
    assert L.flarepp_mix_backward_workspace_size(1, 1, 0, 16, 16, BF16) == 0
    # a token shard with no tokens needs no workspace; otherwise as the encode
    assert L.flare_encode_lse_workspace_size(1, 2, 0, 64, 32, BF16) == 0
    assert L.flare_encode_lse_workspace_size(1, 2, 5000, 64, 32, BF16) == L.flare_encode_workspace_size(
        1, 2, 5000, 64, 32, BF16)


def test_option_hooks_round_trip(L):
    old = L.flare_set_split_override(5)
    assert L.flare_set_split_override(old) == 5
    old = L.flare_set_wait_limit_ms(123)
    assert L.flare_set_wait_limit_ms(old) == 123


def test_header_is_plain_c_and_links(tmp_path):
    """include/flarepp.h compiles as pedantic C99; a C program links against
    libflarepp.so and calls a host-side query (no GPU needed)."""
    import os
    import shutil

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_abi.c"
    src.write_text(
        '#include <stdio.h>\n#include "flarepp.h"\n'
        "int main(void) {\n"
        "  size_t a = flarepp_saved_bytes(1, 16, 256, 64, FLARE_BF16);\n"
        "  size_t b = flarepp_saved_bytes(1, 1, 17, 64, FLARE_BF16);\n"
        '  printf("%zu %zu\\n", a, b);\n'
        "  return 0;\n}\n")
    lib_dir = os.path.dirname(flare.LIB_PATH)
    exe = tmp_path / "use_abi"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                    os.path.dirname(flare.HEADER_PATH), str(src), "-L", lib_dir, "-lflarepp",
                    f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert out == [str(flare.flarepp_saved_bytes(1, 16, 256, 64, 1)), "0"]
