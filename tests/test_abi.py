"""The C header against the Python binding: every field offset and size of the
structures the binding mirrors with ctypes, and every constant it repeats.
A small C program including include/df11.h, built with the host compiler,
prints the header's view.  No GPU needed."""
import ctypes
import os
import shutil
import subprocess

import pytest


@pytest.fixture(scope="module")
def df11():
    from entropy_decoding_b200 import build
    build.build()
    from entropy_decoding_b200 import df11 as mod
    return mod


STRUCTS = {"df11_blob_info": "BlobInfo", "df11_decode_opts": "DecodeOpts", "df11_encode_result": "EncodeResult",
           "df11_rans_tensor_info": "RansTensorInfo", "df11_gemm_matrix": "GemmMatrix"}
CONSTANTS = {
    "DF11_OK": "DF11_OK", "DF11_EINVAL": "DF11_EINVAL", "DF11_ENOMEM": "DF11_ENOMEM", "DF11_ECUDA": "DF11_ECUDA",
    "DF11_ECORRUPT": "DF11_ECORRUPT", "DF11_EUNSUPPORTED": "DF11_EUNSUPPORTED",
    "DF11_BF16": "DF11_BF16", "DF11_FP8_E4M3": "DF11_FP8_E4M3",
    "DF11_DEV_ERR_SPAN": "DEV_ERR_SPAN", "DF11_DEV_ERR_CODE": "DEV_ERR_CODE", "DF11_DEV_ERR_AUX": "DEV_ERR_AUX",
    "DF11_DEV_ERR_TIMEOUT": "DEV_ERR_TIMEOUT", "DF11_DEV_ERR_BOUNDS": "DEV_ERR_BOUNDS",
    "DF11_WALKER_AUTO": "WALKER_AUTO", "DF11_WALKER_WINDOW": "WALKER_WINDOW",
    "DF11_WALKER_BYTE_STEP": "WALKER_BYTE_STEP",
    "DF11_ENCODE_NO_CHUNK_COUNTS": "ENCODE_NO_CHUNK_COUNTS",
    "DF11_NOALLOC_SCRATCH_BYTES": "NOALLOC_SCRATCH_BYTES", "DF11_NOALLOC_MAX_ELEMS": "NOALLOC_MAX_ELEMS",
    "DF11_RANS_TILE_DEFAULT": "RANS_TILE_DEFAULT",
    "DF11_GEMM_TILE_N": "GEMM_TILE_N", "DF11_GEMM_TILE_K": "GEMM_TILE_K", "DF11_GEMM_MAX_MATS": "GEMM_MAX_MATS",
    "DF11_GEMM_MAX_BATCH": "GEMM_MAX_BATCH",
}


def _header_view(df11, tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "df11.h"', "int main(void) {"]
    for cname, pyname in STRUCTS.items():
        for field, _ in getattr(df11, pyname)._fields_:
            lines.append(f'  printf("{cname} {field} %zu %zu\\n", offsetof({cname}, {field}), '
                         f"sizeof((({cname} *)0)->{field}));")
        lines.append(f'  printf("{cname} sizeof %zu 0\\n", sizeof({cname}));')
    for cname in CONSTANTS:
        lines.append(f'  printf("const {cname} %llu 0\\n", (unsigned long long)({cname}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "abi.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "abi"
    include = os.path.join(os.path.dirname(df11.HEADER_PATH))
    subprocess.run([cc, "-std=c11", "-Wall", "-Werror", "-I", include, str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    view = {}
    for line in out.splitlines():
        a, b, c, d = line.split()
        view[(a, b)] = (int(c), int(d))
    return view


def test_structures_and_constants_match_the_header(df11, tmp_path):
    view = _header_view(df11, tmp_path)
    for cname, pyname in STRUCTS.items():
        cls = getattr(df11, pyname)
        for field, ctype in cls._fields_:
            off, size = view[(cname, field)]
            assert getattr(cls, field).offset == off, (cname, field)
            assert ctypes.sizeof(ctype) == size, (cname, field)
        assert ctypes.sizeof(cls) == view[(cname, "sizeof")][0], cname
        # every field of the C structure is mirrored: the sizes add up
        assert sum(ctypes.sizeof(t) for _, t in cls._fields_) <= ctypes.sizeof(cls)
    for cname, pyname in CONSTANTS.items():
        assert view[("const", cname)][0] == getattr(df11, pyname), cname
