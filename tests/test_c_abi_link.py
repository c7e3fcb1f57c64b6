"""The boundary from plain C: include/kda.h compiles as strict C99 (no C++ in the header), a C
program that takes the address of every declared entry point links against libkda.so, and its
host-only calls (status strings, version) run without a GPU."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

from kimi_delta_attention_32_b200 import build as kbuild
from test_abi import ROOT, declared_functions


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_links_every_entry_point(tmp_path):
    lib = kbuild.build()
    names = declared_functions()
    src = ["#include <stdio.h>", "#include <string.h>", '#include "kda.h"',
           "typedef void (*any_fn)(void);",
           "static const any_fn entry_points[] = {"]
    src += [f"    (any_fn){n}," for n in names]
    src += ["};",
            "int main(void) {",
            "    size_t i;",
            "    for (i = 0; i < sizeof entry_points / sizeof entry_points[0]; ++i)",
            "        if (entry_points[i] == NULL) return 2;",
            '    if (strcmp(kda_status_string(KDA_OK), "ok") != 0) return 3;',
            "    if (kda_version() < 100) return 4;",
            '    printf("%d entry points\\n", (int)(sizeof entry_points / sizeof entry_points[0]));',
            "    return 0;",
            "}"]
    c_file = tmp_path / "abi.c"
    c_file.write_text("\n".join(src) + "\n")
    exe = tmp_path / "abi"
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), str(c_file), "-L", libdir, "-lkda",
           f"-Wl,-rpath,{libdir}", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == f"{len(names)} entry points"
