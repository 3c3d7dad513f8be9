"""The C ABI library loads on a machine without a GPU, exports every function
include/ab.h declares, and rejects bad arguments on the host before any CUDA
call (no compute call is made here)."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_queries_b200 as ab
from block_sparse_attention_queries_b200 import build as abbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    abbuild.build()
    return ab.lib()


def _declared():
    txt = open(os.path.join(ROOT, "include", "ab.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(ab_\w+)\s*\(", txt, flags=re.M)))


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert set(declared) == set(ab.EXPORTS), declared
    for name in declared:
        assert hasattr(lib, name), name


def test_budget_and_workspace(lib):
    p = ab.Params(B=1, H=40, L=32760, d=128, q_block=128, kv_block=16, C=8, keep_ratio=0.11)
    assert ab.budget(p) == 225
    assert ab.budget(ab.Params(B=1, H=24, L=118800, d=128, keep_ratio=0.08)) == 594
    assert ab.budget(ab.Params(B=1, H=1, L=1024, d=64, q_block=64, C=4, keep_ratio=0.10)) == 6
    ws = ab.workspace_size(p)
    # K summaries + bf16 centroids + counts
    assert ws >= 40 * 2048 * 128 * 2 + 40 * 256 * 8 * 128 * 2 + 40 * 256 * 8 * 4


@pytest.mark.parametrize("field,value,status", [
    ("d", 96, 2), ("d", 0, 1), ("q_block", 32, 2), ("kv_block", 8, 2), ("kv_block", 0, 1),
    ("C", 3, 2), ("C", 0, 1), ("C", 17, 1), ("kmeans_iters", 0, 1), ("keep_ratio", 0.0, 1),
    ("keep_ratio", 1.5, 1), ("L", 0, 1), ("B", 0, 1), ("L", 2**24 + 1, 1),
])
def test_invalid_params_rejected_on_host(lib, field, value, status):
    kw = dict(B=1, H=2, L=1000, d=128, q_block=128, kv_block=16, C=8, keep_ratio=0.1)
    kw[field] = value
    p = ab.Params(**kw).c()
    n = ctypes.c_size_t(0)
    assert lib.ab_workspace_size(ctypes.byref(p), ctypes.byref(n)) == status
    assert lib.ab_budget(ctypes.byref(p)) == -1


def test_null_and_misaligned_pointers_rejected(lib):
    p = ab.Params(B=1, H=1, L=256, d=64, q_block=64, kv_block=16, C=4).c()
    # null pointers
    assert lib.ab_select(ctypes.byref(p), None, None, None, None, None, None, 0, None) == 1
    assert lib.ab_sample(ctypes.byref(p), None, None, None, None, None) == 1
    assert lib.ab_attention(ctypes.byref(p), None, None, None, None, None, None, None, None) == 1
    assert lib.ab_attention_dense(ctypes.byref(p), None, None, None, None, None) == 1
    # misaligned (never dereferenced: rejected before any launch)
    bad = ctypes.c_void_p(0x1000 + 8)
    good = ctypes.c_void_p(0x1000)
    assert lib.ab_attention_dense(ctypes.byref(p), bad, good, good, good, None) == 1
    # workspace too small
    assert lib.ab_select(ctypes.byref(p), good, good, good, None, None, good, 16, None) == 6


def test_status_strings(lib):
    for s in range(7):
        assert lib.ab_status_string(s)
    assert ab.status_string(6) == "workspace too small"


def test_params_struct_matches_the_header(tmp_path):
    """The ctypes mirror of ab_params has the C struct's size and offsets."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    names = [n for n, _ in ab.ab_params._fields_]
    src = tmp_path / "layout.c"
    src.write_text("#include <stdio.h>\n#include <stddef.h>\n#include \"ab.h\"\nint main(void) {\n"
                   + "".join(f'  printf("%zu\\n", offsetof(ab_params, {n}));\n' for n in names)
                   + '  printf("%zu\\n", sizeof(ab_params));\n  return 0;\n}\n')
    exe = tmp_path / "layout"
    subprocess.check_call([cc, "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)])
    got = [int(x) for x in subprocess.check_output([str(exe)]).split()]
    want = [getattr(ab.ab_params, n).offset for n in names] + [ctypes.sizeof(ab.ab_params)]
    assert got == want


def test_key_length_field(lib):
    # cross-attention: Nkv follows L_kv, Nq follows L
    p = ab.Params(B=1, H=3, L=8192, d=128, q_block=128, kv_block=16, C=8, keep_ratio=0.1, L_kv=3330)
    assert (p.Nq, p.Nkv) == (64, 209)
    assert ab.budget(p) == 21                      # floor(0.1 * 209 + 1/2)
    assert ab.budget(ab.Params(B=1, H=3, L=8192, d=128, keep_ratio=0.1, L_kv=0)) == 51
    ws = ab.workspace_size(p)
    assert ws >= 3 * 209 * 128 * 2 + 3 * 64 * 8 * 128 * 2 + 3 * 64 * 8 * 4
    assert ws < ab.workspace_size(ab.Params(B=1, H=3, L=8192, d=128, keep_ratio=0.1))
    for bad in (-1, 2**24 + 1):
        c = ab.Params(B=1, H=2, L=1000, d=128, L_kv=bad).c()
        n = ctypes.c_size_t(0)
        assert lib.ab_workspace_size(ctypes.byref(c), ctypes.byref(n)) == 1
        assert lib.ab_budget(ctypes.byref(c)) == -1


def test_list_outputs_are_checked_before_any_call():
    import torch
    p = ab.Params(B=1, H=2, L=300, d=64, q_block=64, kv_block=16, C=4)
    P = torch.zeros(1, 2, p.Nq, p.Nkv)
    good = (torch.zeros(1, 2, p.Nq, p.Nkv, dtype=torch.int32), torch.zeros(1, 2, p.Nq, p.Nkv, dtype=torch.int32),
            torch.zeros(1, 2, p.Nq, dtype=torch.int32))
    assert ab._list_outputs(p, P, good)[0] is good[0]
    with pytest.raises(ValueError):
        ab._list_outputs(p, P, (good[0], good[1], torch.zeros(1, 2, p.Nq + 1, dtype=torch.int32)))
    with pytest.raises(ValueError):
        ab._list_outputs(p, P, (good[0].float(), good[1], good[2]))
    with pytest.raises(ValueError):
        ab._list_outputs(p, P.double(), good)


def test_forward_slice_range_checked_on_host(lib):
    # a slice must be a non-empty range of the whole problem's B * H heads;
    # rejected before anything touches the device (pointers never read)
    p = ab.Params(B=2, H=3, L=256, d=64, q_block=64, kv_block=16, C=4).c()
    good = ctypes.c_void_p(0x1000)
    args = (good,) * 8 + (good, ctypes.c_size_t(1 << 30), None)
    for bh0, nbh in ((0, 0), (-1, 2), (5, 2), (0, 7)):
        assert lib.ab_forward_slice(ctypes.byref(p), bh0, nbh, *args) == 1
    assert lib.ab_forward_slice(ctypes.byref(p), 0, 2, good, good, None, *args[3:]) == 1  # V missing


def test_select_sample_checked_on_host(lib):
    # null, misaligned and workspace errors are found before anything is
    # enqueued, both for rows the fused kernel takes (Nkv <= 2048) and for
    # longer rows, which run the two launches (pointers never read)
    good, bad = ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1008)
    for L in (256, 2049 * 16):  # Nkv = 16 and 2049
        p = ab.Params(B=1, H=1, L=L, d=64, q_block=64, kv_block=16, C=4).c()
        big = ctypes.c_size_t(1 << 40)
        assert lib.ab_select_sample(ctypes.byref(p), None, None, None, None, None, None, None, 0, None) == 1
        assert lib.ab_select_sample(ctypes.byref(p), good, good, good, None, good, good, good, big, None) == 1
        assert lib.ab_select_sample(ctypes.byref(p), good, good, good, good, good, bad, good, big, None) == 1
        assert lib.ab_select_sample(ctypes.byref(p), good, good, good, good, good, good, good,
                                    ctypes.c_size_t(16), None) == 6


def test_whole_path_calls_check_every_argument_first(lib):
    # ab_forward, ab_forward_slice and ab_forward_host find a null or
    # misaligned buffer (or a short workspace) before anything is enqueued,
    # whichever buffer it is (pointers never read)
    p = ab.Params(B=1, H=2, L=256, d=64, q_block=64, kv_block=16, C=4).c()
    good, bad = ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1008)
    big, small = ctypes.c_size_t(1 << 40), ctypes.c_size_t(16)
    # Q, K, V, P, idx, pi_q32, count, O, workspace
    for k in range(9):
        for wrong in (None, bad):
            dev = [good] * 9
            dev[k] = wrong
            assert lib.ab_forward(ctypes.byref(p), *dev, big, None) == 1, (k, wrong)
            assert lib.ab_forward_slice(ctypes.byref(p), 0, 1, *dev, big, None) == 1, (k, wrong)
            host = [good] * 4
            assert lib.ab_forward_host(ctypes.byref(p), *host, dev[0], dev[1], dev[2], *dev[3:], big, None) == 1
    dev = [good] * 9
    assert lib.ab_forward(ctypes.byref(p), *dev, small, None) == 6
    assert lib.ab_forward_slice(ctypes.byref(p), 1, 1, *dev, small, None) == 6
    assert lib.ab_forward_host(ctypes.byref(p), None, good, good, good, *dev, big, None) == 1
    assert lib.ab_forward_host(ctypes.byref(p), good, good, good, good, *dev, small, None) == 6
