"""The C ABI from plain C: a C99 program that includes include/kda.h, links
libkda.so and calls the host-side parts of the API (version, status strings,
workspace query, argument validation) compiles without warnings and runs
without a GPU."""
import os
import shutil
import subprocess

import pytest

from gated_delta_rule_60_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "kda.h"

int main(void)
{
    char buf[64];
    void *fake = (void *)(size_t)256;     /* never dereferenced: validation fails first */
    kda_status st;
    printf("version %d\n", (int)kda_version());
    printf("ok '%s'\n", kda_status_string(KDA_OK));
    printf("ws %zu\n", kda_chunk_fwd_workspace_size(1, 1 << 20, 8, 128, 128, KDA_BF16) > 0 ? (size_t)1 : (size_t)0);
    st = kda_chunk_fwd(NULL, fake, fake, fake, fake, NULL, NULL, 1, 32, 2, 16, 16,
                       KDA_FP32, fake, NULL, NULL, 0, NULL);
    printf("null q %d\n", (int)st);
    st = kda_chunk_fwd(fake, fake, fake, fake, fake, NULL, NULL, 1, 32, 2, 48, 48,
                       KDA_FP32, fake, NULL, NULL, 0, NULL);
    printf("d48 %d\n", (int)st);
    st = kda_decode_step(fake, fake, fake, fake, fake, (float *)fake, fake, 0, 2, 16, 16,
                         KDA_FP32, NULL);
    printf("empty decode %d\n", (int)st);
    strncpy(buf, kda_status_string(KDA_ERR_WORKSPACE), sizeof buf - 1);
    buf[sizeof buf - 1] = 0;
    printf("ws '%s'\n", buf);
    return 0;
}
"""


def test_plain_c_program_uses_the_abi(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib = build.build()
    libdir = os.path.dirname(lib)
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "consumer"
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
           "-L", libdir, "-l:libkda.so", "-Wl,-rpath," + libdir]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True,
                         timeout=120).stdout.splitlines()
    assert out[0].startswith("version ") and int(out[0].split()[1]) >= 10000
    assert out[1] == "ok 'ok'"
    assert out[2] == "ws 1"
    assert out[3] == "null q 1"            # KDA_ERR_INVALID_ARGUMENT
    assert out[4] == "d48 2"               # KDA_ERR_UNSUPPORTED
    assert out[5] == "empty decode 0"      # KDA_OK, nothing enqueued
    assert out[6] == "ws 'workspace missing or too small'"
