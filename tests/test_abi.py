"""The C-ABI library loads and exports every entry point include/msa.h declares.
Host-side argument checks return before any CUDA call, so they run without a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

import sparse_attention_routed_b200 as msa

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
HEADER = os.path.join(INCLUDE, "msa.h")


def declared():
    """Every entry point the headers under include/ declare."""
    names = []
    for h in sorted(os.listdir(INCLUDE)):
        if h.endswith(".h"):
            text = re.sub(r"/\*.*?\*/", "", open(os.path.join(INCLUDE, h)).read(), flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(msa_\w+)\s*\(", text, flags=re.M)
    return names


def test_header_declarations_are_exported():
    names = declared()
    assert len(names) >= 10
    assert sorted(names) == sorted(msa.EXPORTED)
    msa.lib()
    lib = ctypes.CDLL(msa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_header_enum_values_match_the_binding():
    """Every enumerator include/msa.h declares has the same value in the Python binding."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    found = {}
    for body in re.findall(r"typedef\s+enum\s*\{(.*?)\}", text, flags=re.S):
        for name, val in re.findall(r"(MSA_\w+)\s*=\s*(\d+)", body):
            found[name] = int(val)
    assert len(found) >= 13
    for name, val in found.items():
        assert getattr(msa, name) == val, name


def test_status_strings():
    for s in range(7):
        assert msa.msa_status_string(s) and msa.msa_status_string(s) != "unknown status"
    assert msa.msa_status_string(99) == "unknown status"


def test_bank_create_rejects_bad_arguments():
    lens = np.array([10, 20], dtype=np.int64)
    fake = 0x10000  # never dereferenced: validation fails first
    cases = [
        dict(n_docs=0, n_kv_heads=1, head_dim=64),
        dict(n_docs=2, n_kv_heads=0, head_dim=64),
        dict(n_docs=2, n_kv_heads=1, head_dim=96),
        dict(n_docs=2, n_kv_heads=1, head_dim=64, route_dim=128),
        dict(n_docs=2, n_kv_heads=1, head_dim=64, rope_base=0.5),
        dict(n_docs=2, n_kv_heads=1, head_dim=64, kv_location=7),
        dict(n_docs=2, n_kv_heads=1, head_dim=64, k=0),
        dict(n_docs=2, n_kv_heads=1, head_dim=64, k=fake + 2),   # misaligned
    ]
    for c in cases:
        kw = dict(doc_lens=lens, k=fake, v=fake)
        kw.update(c)
        st, h = msa.msa_bank_create(kw.pop("n_docs"), kw.pop("n_kv_heads"), kw.pop("head_dim"), check=False, **kw)
        assert st == msa.MSA_ERR_INVALID_ARG and not h, c
    st, h = msa.msa_bank_create(2, 1, 64, np.array([10, 0]), fake, fake, check=False)
    assert st == msa.MSA_ERR_INVALID_ARG and not h
    st, h = msa.msa_bank_create(2, 1, 64, lens, fake, fake, kv_rows=25, check=False)   # rows too short
    assert st == msa.MSA_ERR_INVALID_ARG and not h
    st, h = msa.msa_bank_create(2, 1, 64, lens, fake, fake, dtype=7, check=False)      # no such element type
    assert st == msa.MSA_ERR_INVALID_ARG and not h
    # fp32 banks are device-tier only
    st, h = msa.msa_bank_create(2, 1, 64, lens, fake, fake, kv_location=msa.MSA_KV_PINNED_HOST,
                                dtype=msa.MSA_DTYPE_F32, check=False)
    assert st == msa.MSA_ERR_UNSUPPORTED and not h


def test_null_handles_are_rejected():
    q = msa.make_query(1, 4, 1, 8, 1, 0x10000, 0x10000, 0x10000, 0x10000)
    assert msa.msa_route(None, q, 1, 0, 0x10000, 0, check=False) == msa.MSA_ERR_INVALID_ARG
    assert msa.msa_attend(None, q, 1, 0x10000, 0x10000, check=False) == msa.MSA_ERR_INVALID_ARG
    assert msa.msa_forward(None, q, 1, 0x10000, 0x10000, check=False) == msa.MSA_ERR_INVALID_ARG
    assert msa.msa_build_bank(None, 0, 1, 0x10000, 8, 0, 0, check=False) == msa.MSA_ERR_INVALID_ARG
    assert msa.msa_bank_destroy(None) == msa.MSA_OK


def test_product_path_does_not_import_oracle():
    pkg = os.path.dirname(msa.__file__)
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(root, f), errors="ignore").read()
                assert "oracle" not in re.sub(r"#.*|//.*", "", text).lower().replace("oracle/", ""), f
