"""The C ABI: library loads, exports what include/vsa.h declares, host-side validation.

No test here launches a kernel: descriptors are rejected by host validation
before any CUDA call, and struct layouts are compared with a C probe built by
gcc from the header.
"""
import ctypes
import math
import os
import re
import subprocess
import tempfile

import pytest

import oracle.vsa_oracle as O
import tile_sparse_video_pack_b200 as T
from tile_sparse_video_pack_b200 import vsa as V

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vsa.h")


@pytest.fixture(scope="module")
def lib():
    from tile_sparse_video_pack_b200.build import build
    build()
    return V.library()


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^VSA_API\s+[\w\s\*]+?\b(vsa_\w+)\s*\(", text, re.M)))


def test_header_declares_binding_exports():
    assert header_functions() == sorted(V.EXPORTS)


def header_arity():
    """Parameter count of every function the header declares."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"^VSA_API\s+[\w\s\*]+?\b(vsa_\w+)\s*\(([^)]*)\)", text, re.M):
        params = [x for x in m.group(2).split(",") if x.strip() and x.strip() != "void"]
        out[m.group(1)] = len(params)
    return out


def test_binding_argument_counts_match_header(lib):
    ar = header_arity()
    assert sorted(ar) == header_functions()
    for name, n in ar.items():
        assert len(getattr(lib, name).argtypes) == n, name


def test_library_exports_every_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", V.LIB_PATH], capture_output=True, text=True, check=True)
    syms = {ln.split()[-1] for ln in out.stdout.splitlines() if " T " in ln}
    for name in header_functions():
        assert name in syms, name
        assert getattr(lib, name) is not None


def test_struct_layouts_match_c(lib):
    src = r"""
#include <stdio.h>
#include <stddef.h>
#include "vsa.h"
int main(void) {
  printf("%zu %zu %zu\n", sizeof(vsa_desc), sizeof(vsa_plan_info), sizeof(vsa_plan_stats));
  printf("%zu %zu %zu %zu\n", offsetof(vsa_desc, tile_shape), offsetof(vsa_desc, k_per_head),
         offsetof(vsa_desc, softmax_scale), offsetof(vsa_plan_info, workspace_bytes));
  return 0;
}
"""
    with tempfile.TemporaryDirectory() as d:
        c, exe = os.path.join(d, "p.c"), os.path.join(d, "p")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-std=c99", "-I", os.path.dirname(HEADER), c, "-o", exe], check=True)
        lines = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    sizes = [int(x) for x in lines[0].split()]
    offs = [int(x) for x in lines[1].split()]
    assert sizes == [ctypes.sizeof(V.VsaDesc), ctypes.sizeof(V.VsaPlanInfo), ctypes.sizeof(V.VsaPlanStats)]
    assert offs == [V.VsaDesc.tile_shape.offset, V.VsaDesc.k_per_head.offset, V.VsaDesc.softmax_scale.offset,
                    V.VsaPlanInfo.workspace_bytes.offset]


def test_k_from_sparsity_matches_oracle_rule(lib):
    for n in (1, 4, 7, 120, 1680, 1920, 3600):
        for s in [i / 40 for i in range(41)] + [0.95, 0.9, 0.75, 0.333]:
            assert T.k_from_sparsity(s, n) == O.k_from_sparsity(s, n), (s, n)
    assert T.k_from_sparsity(-0.1, 10) == 0 and T.k_from_sparsity(1.5, 10) == 0
    assert T.k_from_sparsity(math.nan, 10) == 0 and T.k_from_sparsity(0.5, 0) == 0


def status_string(lib, s):
    return lib.vsa_status_string(s).decode()


def test_status_strings(lib):
    for s, name in V.STATUS_NAMES.items():
        assert status_string(lib, s).startswith(name)


def _desc(**over):
    base = dict(batch=1, heads=2, head_dim=64, T=4, H=8, W=8, segments=(64, 64),
                tile_shapes=((4, 4, 4), (4, 4, 4)), k_per_head=(2, 2))
    base.update(over)
    return V.make_desc(**base)


BAD = {
    "head_dim": dict(head_dim=96),
    "heads0": dict(heads=0, tile_shapes=(), k_per_head=()),
    "tile_product": dict(tile_shapes=((4, 4, 4), (4, 4, 2))),
    "tile_zero": dict(tile_shapes=((4, 4, 4), (0, 8, 8))),
    "k_zero": dict(k_per_head=(0, 2)),
    "k_too_big": dict(k_per_head=(2, 5)),
    "grid": dict(T=0),
    "batch": dict(batch=0),
    "segment": dict(segments=(64, 0)),
    "proj": dict(proj_dim=32),
    "score_mode": dict(score_mode=7),
    "tripool_proj": dict(score_mode="tripool", proj_dim=12),
    "tripool_proj_small": dict(score_mode="tripool", proj_dim=4),
    "tripool_proj_big": dict(score_mode="tripool", proj_dim=264),
    "scale": dict(softmax_scale=-1.0),
    # R2VA budgets: segment 1 (64 tokens, one tile) may be marked as a reference stream
    "seg_ref_value": dict(seg_ref=(0, 2), k_ref_per_head=(1, 1)),
    "seg_ref_past_segments": dict(seg_ref=(0, 0, 1), k_ref_per_head=(1, 1)),
    "k_ref_zero": dict(seg_ref=(0, 1), k_ref_per_head=(0, 1)),
    "k_ref_too_big": dict(seg_ref=(0, 1), k_ref_per_head=(1, 2)),
    "k_ref_without_reference": dict(k_ref_per_head=(1, 1)),
}


@pytest.mark.parametrize("case", sorted(BAD))
def test_plan_rejects_bad_descriptor(lib, case):
    h = ctypes.c_void_p(1234)
    st = lib.vsa_plan_create(ctypes.byref(_desc(**BAD[case])), ctypes.byref(h))
    assert st == 1, (case, V.STATUS_NAMES.get(st))
    assert not h.value


@pytest.mark.parametrize("over", [{}, dict(seg_ref=(0, 1), k_ref_per_head=(1, 1)),
                                  dict(score_mode="tripool", proj_dim=8),
                                  dict(score_mode="tripool", proj_dim=256)])
def test_plan_accepts_good_descriptor(lib, over):
    """A valid descriptor passes host validation: with no GPU the create fails only at its
    first CUDA call; with one it succeeds."""
    h = ctypes.c_void_p()
    st = lib.vsa_plan_create(ctypes.byref(_desc(**over)), ctypes.byref(h))
    assert st in (0, 3, 6), V.STATUS_NAMES.get(st)      # OK, CUDA or NO_MEMORY, never INVALID_ARG
    if st == 0:
        assert h.value
        assert lib.vsa_plan_destroy(h) == 0
    else:
        assert not h.value


def test_null_arguments(lib):
    h = ctypes.c_void_p()
    assert lib.vsa_plan_create(None, ctypes.byref(h)) == 1
    assert lib.vsa_plan_create(ctypes.byref(_desc()), None) == 1
    assert lib.vsa_plan_destroy(None) == 0
    assert lib.vsa_tile_pack(None, None, None, None, None, None, None, None) == 1
    assert lib.vsa_sparse_attn(None, None, None, None, None, None, None, None, None) == 1
    assert lib.vsa_plan_check(None) == 1
    assert lib.vsa_plan_query(None, None) == 1


def test_every_compute_call_rejects_a_null_plan(lib):
    """A NULL plan (with every other pointer NULL) is an argument error, returned before any
    CUDA call, for every entry point that takes a plan."""
    ar = header_arity()
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    for name, n in ar.items():
        m = re.search(r"\b" + name + r"\s*\(([^)]*)\)", text)
        first = m.group(1).split(",")[0]
        if "vsa_plan*" not in first.replace(" ", "") or name in ("vsa_plan_destroy",):
            continue
        f = getattr(lib, name)
        # NULL for pointers, 0 for integer arguments
        args = [0 if t in (ctypes.c_int32, ctypes.c_uint64, ctypes.c_int64, ctypes.c_double) else None
                for t in f.argtypes]
        assert len(args) == n, name
        assert f(*args) == 1, name   # VSA_ERR_INVALID_ARG
