"""The C ABI used from C and C++, without a GPU: both headers compile as
strict C99 and C++17 with warnings as errors, and a C program linked against
libnvfp4.so gets the size helpers, the status strings and the host-side
argument validation (which returns before any device work)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
LIBDIR = os.path.join(ROOT, "w4a4_gemm_nvfp4_b200")


@pytest.fixture
def scratch():
    """A scratch folder inside the repository's (git-ignored) build folder."""
    import pathlib

    d = pathlib.Path(ROOT, "_build", "c_abi_test", str(os.getpid()))
    d.mkdir(parents=True, exist_ok=True)
    yield d
    shutil.rmtree(d, ignore_errors=True)


PROGRAM = r"""
#include <stdio.h>
#include <string.h>

#include "nvfp4.h"
#include "nvfp4_testing.h"

int main(void) {
  /* 256 x 512: 256 * 256 code bytes; 130 rows pad to 256 scale rows of 32 bytes */
  if (nvfp4_codes_bytes(256, 512) != (size_t)256 * 256) return 1;
  if (nvfp4_scales_bytes(130, 512) != (size_t)256 * 32) return 2;
  if (nvfp4_gemm_workspace_bytes() == 0) return 3;
  if (nvfp4_quantize_workspace_bytes(130, 512) < nvfp4_gemm_workspace_bytes()) return 4;
  {
    nvfp4_status st = nvfp4_quantize(NULL, 128, 512, 512, NVFP4_MODE_SIX, NVFP4_RULE_MAX, 448.0f,
                                     NULL, NULL, NULL, NULL, 0, NULL);
    if (st != NVFP4_ERR_INVALID_ARG) return 5;
    if (strlen(nvfp4_last_error_message()) == 0) return 6;
  }
  {
    char buf[64];
    nvfp4_status st = nvfp4_gemm(buf, buf, NULL, buf, buf, NULL, 64, 64, 100, buf, 64,
                                 NVFP4_OUT_BF16, buf, sizeof(buf), NULL);
    if (st != NVFP4_ERR_INVALID_ARG) return 7;
  }
  if (strcmp(nvfp4_status_string(NVFP4_ERR_TIMEOUT), "NVFP4_ERR_TIMEOUT") != 0) return 8;
  nvfp4_testing_set_gemm_wait(0, 0);
  printf("ok\n");
  return 0;
}
"""


def _compiler(name):
    path = shutil.which(name)
    if path is None:
        pytest.skip(f"{name} not found")
    return path


@pytest.mark.parametrize("lang", ["c99", "c++17"])
def test_headers_compile_strictly(lang, scratch):
    cc = _compiler("gcc" if lang == "c99" else "g++")
    src = scratch / ("t.c" if lang == "c99" else "t.cc")
    src.write_text('#include "nvfp4.h"\n#include "nvfp4_testing.h"\nint main(void) { return 0; }\n')
    subprocess.run([cc, f"-std={lang}", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", INCLUDE,
                    "-fsyntax-only", str(src)], check=True, capture_output=True)


def test_c_program_links_and_validates_on_the_host(scratch):
    lib = os.path.join(LIBDIR, "libnvfp4.so")
    if not os.path.exists(lib):
        pytest.skip("libnvfp4.so is not built")
    cc = _compiler("gcc")
    src = scratch / "abi.c"
    src.write_text(PROGRAM)
    exe = scratch / "abi"
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", INCLUDE, str(src), "-L", LIBDIR, "-lnvfp4",
                    f"-Wl,-rpath,{LIBDIR}", "-o", str(exe)], check=True, capture_output=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.strip() == "ok"
