"""The C ABI from C: tests/abi_client.c is compiled against include/wvae.h alone
(strict C99, warnings as errors; and again as C++17, through the header's
extern "C" block), linked with libwvae.so and run without a GPU."""
import os
import shutil
import subprocess

import pytest

from video_diffusion_vae_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "abi_client.c")
LIBDIR = os.path.dirname(B.LIB_PATH)

EXPECTED = {
    "version": str(1 << 16),
    "status0": "ok",
    # prepacked 3x3x3 512->512 bf16: [cout][27 taps][cin] bf16 + fp32 bias
    "conv_packed_512x512x27_bf16": str(512 * 27 * 512 * 2 + 512 * 4),
    "conv_packed_unsupported": "0",
    # the two bf16 activation tensors A1, A2 of a 256->256 block at [4,176,312]
    "resblock_ws_256_bf16": str(2 * 4 * 176 * 312 * 256 * 2),
    "trunk_launches": "22",
    "norm_null_x": "1",        # WVAE_ERR_INVALID_ARG
    "norm_bad_c": "2",         # WVAE_ERR_UNSUPPORTED (C % 8)
    "norm_misaligned": "3",    # WVAE_ERR_ALIGNMENT
    "selftest_bad_limit": "1",
}


def _compiler(lang):
    return shutil.which("gcc" if lang == "c" else "g++")


@pytest.mark.parametrize("lang", ["c", "c++"])
def test_c_client_against_header_and_library(tmp_path, lang):
    cc = _compiler(lang)
    if cc is None:
        pytest.skip(f"no {lang} compiler")
    if not os.path.exists(B.LIB_PATH):
        pytest.skip("libwvae.so not built")
    exe = str(tmp_path / "abi_client")
    std = ["-std=c99", "-pedantic"] if lang == "c" else ["-x", "c++", "-std=c++17"]
    subprocess.check_call([cc, *std, "-Wall", "-Wextra", "-Werror",
                           "-I", os.path.join(ROOT, "include"), SRC,
                           "-L", LIBDIR, "-lwvae", f"-Wl,-rpath,{LIBDIR}", "-o", exe])
    out = subprocess.run([exe], capture_output=True, text=True, timeout=60, check=True).stdout
    got = dict(line.split(" ", 1) for line in out.strip().splitlines())
    for k, v in EXPECTED.items():
        assert got[k] == v, (k, got[k], v)
    # every status has a name, and the names differ
    names = [got[f"status{s}"] for s in range(8)]
    assert all(names) and len(set(names)) == 8
