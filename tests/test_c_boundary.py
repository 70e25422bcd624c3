"""The boundary as a C program sees it: include/w4a4.h compiles as plain C11
(no C++ or torch types), and a program that takes the address of every
function it declares links against the built library and runs its host-side
checks (no GPU needed: only argument validation and empty problems)."""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a4.h")


def declared_functions():
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in {"if", "defined"}))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_header_is_plain_c_and_links(tmp_path):
    from bit_diffusion_transformer_nvfp4_b200 import build
    lib = build.build()
    names = declared_functions()
    refs = "\n".join(f"  (entry)&{n}," for n in names)
    prog = f"""
#include <stdio.h>
#include "w4a4.h"
typedef void (*entry)(void);
static const entry every_entry[] = {{
{refs}
}};
int main(void) {{
  int bad = 0;
  for (unsigned i = 0; i < sizeof every_entry / sizeof every_entry[0]; ++i) bad += every_entry[i] == 0;
  /* host-side checks only: a zero K, an empty problem, a bad enum */
  if (nvfp4_sf_bytes(128, 0) != 0) ++bad;
  if (nvfp4_sf_bytes(128, 64) != (size_t)128 * 4) ++bad;
  if (w4a4_gemm(0, 0, 0, 0, 0, 256, 256, 0, 0, 0, 0, 0, 0, W4A4_EPI_NONE, 0, 256, 0) != W4A4_OK) ++bad;
  if (w4a4_gemm(0, 0, 0, 0, 16, 256, 250, 0, 0, 0, 0, 0, 0, W4A4_EPI_NONE, 0, 256, 0) != W4A4_ERR_SHAPE) ++bad;
  if (fp8_quantize(0, 16, 16, 16, 3, 0, 16, 0, 0, 0, 0) != W4A4_ERR_ARG) ++bad;
  printf("%u entries, %d bad\\n", (unsigned)(sizeof every_entry / sizeof every_entry[0]), bad);
  return bad;
}}
"""
    c = tmp_path / "boundary.c"
    c.write_text(prog)
    exe = tmp_path / "boundary"
    libdir = os.path.dirname(lib)
    cuda_lib = "/usr/local/cuda/lib64"
    res = subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-pedantic", f"-I{os.path.join(ROOT, 'include')}",
                          str(c), "-o", str(exe), f"-L{libdir}", "-l:libw4a4.so", f"-Wl,-rpath,{libdir}",
                          f"-Wl,-rpath,{cuda_lib}"], capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert f"{len(names)} entries, 0 bad" in run.stdout
