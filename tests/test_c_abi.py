"""The boundary is a C ABI: a strict C99 program (warnings as errors) can
include include/gptoss.h and link against libgptoss_attn.so, taking the
address of every function the header declares.  The link resolves each
symbol with C linkage; nothing is run (no GPU here)."""

import os
import re
import shutil
import subprocess

import pytest

from attention_yarn_rope_b200 import build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "gptoss.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gptoss_\w+)\s*\(", src)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_compiles_as_c99_and_links(tmp_path):
    lib = build_lib.build()
    names = _declared()
    body = "\n".join(f"    (entry)&{n}," for n in names)
    c_src = tmp_path / "use_gptoss.c"
    c_src.write_text(f"""#include "gptoss.h"

typedef void (*entry)(void);

int main(void) {{
  static const entry entries[] = {{
{body}
  }};
  gptoss_rope_params rope = {{150000.0, 32.0, 4096, 64, 1.0, 32.0}};
  gptoss_strides strides = {{0, 0, 64}};
  (void)rope;
  (void)strides;
  return entries[0] == 0;
}}
""")
    exe = tmp_path / "use_gptoss"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), str(c_src),
           "-L", os.path.dirname(lib), "-lgptoss_attn", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert exe.exists()
