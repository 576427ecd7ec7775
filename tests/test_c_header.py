"""include/tpa.h is a C header: a C99 translation unit that includes it and takes the address
of every declared entry point compiles with gcc -Wall -Werror and links against libtpa.so, and
its host-side checks answer a C caller (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

from factorized_kv_cache_b200 import tpa as T

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc is not installed")
def test_header_compiles_as_c99_and_links(tmp_path):
    names = T.declared_functions()
    src = tmp_path / "uses_tpa.c"
    body = "\n".join(f"  fns[{k}] = (void (*)(void))&{n};" for k, n in enumerate(names))
    src.write_text(f"""#include "tpa.h"
#include <stdio.h>
int main(void) {{
  void (*fns[{len(names)}])(void);
{body}
  tpa_cache c = {{0}};
  c.batch = 1;
  tpa_step_plan plan = {{{{0}}}};
  /* a plan that was never initialised is refused without touching the device */
  if (tpa_step_plan_run(NULL, NULL) != TPA_ERR_NULL || tpa_step_plan_run(&plan, NULL) != TPA_ERR_SHAPE) return 2;
  printf("%zu %d\\n", tpa_factor_elements_per_token(32, 128, 1, 1), (int)(fns[0] != 0) + c.batch);
  return 0;
}}
""")
    exe = tmp_path / "uses_tpa"
    lib_dir = os.path.dirname(T.LIB_PATH)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), "-L", lib_dir, "-ltpa", f"-Wl,-rpath,{lib_dir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    assert out.stdout.split()[0] == "320"      # (R_K+R_V)(h+d_h) at h=32, d_h=128, R=1 (section 关键设计)
