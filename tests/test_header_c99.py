"""include/msa.h is a plain C99 header: a C translation unit that includes it and
names every entry point compiles with -std=c99 -pedantic -Werror, links against
libmsa.so, and runs the calls that need no GPU (status strings, argument checks
that return before any CUDA call)."""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msa.h")
LIBDIR = os.path.join(ROOT, "sparse_attention_routed_b200")


def _declared():
    names = []
    for h in sorted(os.listdir(os.path.dirname(HEADER))):
        if h.endswith(".h"):
            text = re.sub(r"/\*.*?\*/", "", open(os.path.join(os.path.dirname(HEADER), h)).read(), flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(msa_\w+)\s*\(", text, flags=re.M)
    return names


PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "msa.h"
#include "msa_selftest.h"

typedef void (*any_fn)(void);

int main(void) {
  /* every declared entry point, by address: the prototypes are valid C99 */
  any_fn fns[] = { %(fns)s };
  msa_bank_config cfg;
  msa_bank* bank = (msa_bank*)0;
  msa_query q;
  int64_t lens[2] = {10, 20};
  size_t i;
  for (i = 0; i < sizeof(fns) / sizeof(fns[0]); ++i)
    if (!fns[i]) return 10;
  if (strcmp(msa_status_string(MSA_OK), "ok") != 0) return 11;
  if (msa_bank_create((const msa_bank_config*)0, &bank) != MSA_ERR_INVALID_ARG || bank) return 12;
  memset(&cfg, 0, sizeof(cfg));
  cfg.n_docs = 2; cfg.n_kv_heads = 1; cfg.head_dim = 96; cfg.route_dim = 96;
  cfg.doc_lens = lens; cfg.rope_base = 10000.0f;
  if (msa_bank_create(&cfg, &bank) != MSA_ERR_INVALID_ARG || bank) return 13;  /* head_dim 96 */
  memset(&q, 0, sizeof(q));
  if (msa_route((msa_bank*)0, &q, 1, (float*)0, (int32_t*)0, (float*)0, (void*)0) != MSA_ERR_INVALID_ARG) return 14;
  if (msa_route_noalloc((msa_bank*)0, &q, 1, (float*)0, (int32_t*)0, (float*)0, (void*)0) != MSA_ERR_INVALID_ARG)
    return 15;
  if (msa_bank_destroy((msa_bank*)0) != MSA_OK) return 16;
  printf("c99 ok %%u\n", (unsigned)(sizeof(fns) / sizeof(fns[0])));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_header_compiles_as_c99_and_links(tmp_path):
    names = _declared()
    assert len(names) >= 20
    src = tmp_path / "use_msa.c"
    src.write_text(PROGRAM % {"fns": ", ".join(f"(any_fn){n}" for n in names)})
    exe = tmp_path / "use_msa"
    lib = os.path.join(LIBDIR, "libmsa.so")
    assert os.path.exists(lib), "libmsa.so is not built"
    # function pointer -> any_fn casts are valid C; -Wno-cast-function-type keeps
    # -Wextra from flagging the deliberate signature erasure
    cmd = ["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-Wno-cast-function-type",
           "-I" + os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L" + LIBDIR, "-lmsa",
           "-Wl,-rpath," + LIBDIR]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, f"exit {r.returncode}: {r.stdout}{r.stderr}"
    assert r.stdout.strip() == f"c99 ok {len(names)}"
