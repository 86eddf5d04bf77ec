"""The header is plain C: a C99 program compiled against include/gqa_decode.h
links the library, calls its host-only entry points, and reports the struct
layouts, which must equal the Python binding's ctypes mirrors (CPU only)."""
import os
import shutil
import subprocess

import pytest

import gqa_decode_attention_attend_b200 as gqa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PARAMS = ["struct_size", "q", "q_dtype", "k", "v", "kv_dtype", "offsets", "batch", "max_len",
          "max_seq_len", "num_heads", "num_kv_heads", "head_dim", "score_scale", "carry_in",
          "state_out", "out", "out_dtype", "partials_out", "num_splits", "workspace",
          "workspace_bytes", "bias", "flags"]
CODES = ["k_codes", "v_codes", "words", "k_atoms", "v_atoms", "n_atoms"]

PROGRAM = r"""
#include <stddef.h>
#include <stdio.h>
#include "gqa_decode.h"

int main(void) {
  int32_t chunk = 0, splits = 0;
  gqa_decode_params p = {0};
  printf("sizeof params %zu\n", sizeof(gqa_decode_params));
  printf("sizeof codes %zu\n", sizeof(gqa_kv_codes));
  printf("sizeof state %zu\n", sizeof(gqa_state));
@PARAMS@
@CODES@
  {
    const gqa_status st = gqa_plan_splits(16, 8, 4096, 16 * 4096, 148, 2, &chunk, &splits);
    printf("plan %d %d %d\n", (int)st, (int)chunk, (int)splits);
  }
  printf("status %s\n", gqa_status_string(GQA_ERR_WORKSPACE));
  printf("version %d\n", (int)gqa_version());
  p.struct_size = 8; /* wrong size: refused on the host, nothing touches a device */
  printf("refuse %d\n", (int)gqa_decode_attend(&p, NULL));
  return 0;
}
"""


@pytest.fixture(scope="module")
def report(tmp_path_factory):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib = gqa.lib_path()
    gqa.load_library()                       # raises if the library was never built
    d = tmp_path_factory.mktemp("cabi")
    src = d / "prog.c"
    params = "\n".join(f'  printf("params.{f} %zu\\n", offsetof(gqa_decode_params, {f}));' for f in PARAMS)
    codes = "\n".join(f'  printf("codes.{f} %zu\\n", offsetof(gqa_kv_codes, {f}));' for f in CODES)
    src.write_text(PROGRAM.replace("@PARAMS@", params).replace("@CODES@", codes))
    exe = d / "prog"
    libdir = os.path.dirname(lib)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    f"-I{os.path.join(ROOT, 'include')}", str(src), f"-L{libdir}", "-lgqa_decode",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    rep = {}
    for line in out.splitlines():
        key, _, val = line.partition(" ")
        if key == "sizeof":
            k2, v2 = val.split()
            rep["sizeof " + k2] = int(v2)
        else:
            rep[key] = val
    return rep


def test_struct_layouts_match_the_binding(report):
    import ctypes
    assert report["sizeof params"] == ctypes.sizeof(gqa._CParams)
    assert report["sizeof codes"] == ctypes.sizeof(gqa._CCodes)
    assert report["sizeof state"] == ctypes.sizeof(gqa._CState)
    for f in PARAMS:
        assert int(report[f"params.{f}"]) == getattr(gqa._CParams, f).offset, f
    for f in CODES:
        assert int(report[f"codes.{f}"]) == getattr(gqa._CCodes, f).offset, f


def test_host_entry_points_from_c(report):
    status, chunk, splits = (int(x) for x in report["plan"].split())
    assert status == 0 and (chunk, splits) == gqa.gqa_plan_splits(16, 8, 4096, 16 * 4096, 148, 2)
    assert report["status"] == "GQA_ERR_WORKSPACE"
    assert int(report["version"]) == gqa.gqa_version()
    assert int(report["refuse"]) == gqa.GQA_ERR_INVALID_ARGUMENT
