"""The C-ABI library loads and exports every entry point its header declares;
host-side argument checks reject bad calls before anything is launched (no
compute call here, so this runs without a GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dfsattn.h")


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(dfs_[a-z_]+)\s*\(", txt)))


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_36_b200 import dfsattn
    return dfsattn


def test_header_lists_the_path_calls():
    names = _declared()
    for n in ("dfs_hilbert_perm", "dfs_block_score", "dfs_select_mask", "dfs_sparse_attn_fwd", "dfs_unperm"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    so = lib._LIB_PATH
    out = subprocess.run(["nm", "-D", "--defined-only", so], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(dfs_\w+)", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    for n in _declared():
        assert hasattr(lib.LIB, n)
    assert set(lib.EXPORTS) <= set(_declared())


def test_status_strings_and_version(lib):
    assert lib.LIB.dfs_status_string(0) == b"ok"
    assert lib.LIB.dfs_status_string(-3).startswith(b"tensor pointer")
    assert lib.dfs_version() == 100


def test_workspace_bytes(lib):
    s = lib.Shape(1, 12, 128, 21, 30, 52, 128, 32)
    assert lib.dfs_workspace_bytes(s) == 2 * 12 * 1024 * 128 * 4
    bad = lib.Shape(1, 12, 96, 21, 30, 52, 128, 32)          # D = 96 unsupported
    assert lib.dfs_workspace_bytes(bad) == 0
    assert lib.dfs_workspace_bytes(s, which=7) == 0


def _shape_c(lib, **kw):
    base = dict(B=1, nh=2, D=64, T=8, H=16, W=16, blk=64, sb=16)
    base.update(kw)
    return lib._Shape(*[base[n] for n in ("B", "nh", "D", "T", "H", "W", "blk", "sb")])


def test_argument_errors_need_no_gpu(lib):
    L = lib.LIB
    P = ctypes.c_void_p
    fake = P(1 << 20)                      # never dereferenced: checks fail first
    odd = P((1 << 20) + 2)
    sh = _shape_c(lib)
    assert L.dfs_hilbert_perm(None, 1, fake, fake, 1, None, None, None, None, None, None, None) == -1
    assert L.dfs_hilbert_perm(ctypes.byref(sh), 5, fake, fake, 1, None, None, None, None, None, None, None) == -1
    assert L.dfs_hilbert_perm(ctypes.byref(sh), 1, fake, fake, 0, fake, None, None, None, None, None, None) == -1
    assert L.dfs_hilbert_perm(ctypes.byref(sh), 1, fake, fake, 0, odd, None, None, fake, None, None, None) == -3
    bad_d = _shape_c(lib, D=80)
    assert L.dfs_unperm(ctypes.byref(bad_d), fake, fake, fake, None) == -2
    bad_sb = _shape_c(lib, sb=24)
    assert L.dfs_block_score(ctypes.byref(bad_sb), fake, fake, 0.0, fake, fake, 1 << 30, None) == -1
    r16 = _shape_c(lib, sb=4)   # blk / sb = 16 is not supported
    assert L.dfs_block_score(ctypes.byref(r16), fake, fake, 0.0, fake, fake, 1 << 30, None) == -2
    assert L.dfs_block_score(ctypes.byref(sh), fake, fake, 0.0, fake, fake, 16, None) == -6
    prm = lib.select_params("topk", k=9)
    assert L.dfs_select_mask(ctypes.byref(sh), fake, ctypes.byref(prm), fake, fake, 8, None) == -1
    prm = lib.select_params("threshold", cap=-1, tau=0.9)
    assert L.dfs_select_mask(ctypes.byref(sh), fake, ctypes.byref(prm), fake, fake, 8, None) == -1
    prm = lib.select_params(7)
    assert L.dfs_select_mask(ctypes.byref(sh), fake, ctypes.byref(prm), fake, fake, 8, None) == -1
    assert L.dfs_sparse_attn_fwd(ctypes.byref(sh), fake, fake, fake, fake, fake, 0, 0.0, fake, None, None) == -1
    assert L.dfs_sparse_attn_fwd(ctypes.byref(sh), fake, fake, odd, fake, fake, 4, 0.0, fake, None, None) == -3
    zero = _shape_c(lib, T=0)
    assert L.dfs_unperm(ctypes.byref(zero), fake, fake, fake, None) == -1


def test_argument_errors_of_later_entry_points(lib):
    """Extended forward, work order, frame-exact LVSA, backward, no-alloc
    scoring and the workspace query: host-side checks only."""
    L = lib.LIB
    P = ctypes.c_void_p
    fake = P(1 << 20)
    odd = P((1 << 20) + 2)
    sh = _shape_c(lib)                     # blk 64
    sh128 = _shape_c(lib, blk=128)
    opts = lib._AttnOpts(None, None)
    assert L.dfs_sparse_attn_fwd_ex(ctypes.byref(sh), fake, fake, fake, fake, fake, 0, 0.0, ctypes.byref(opts),
                                    fake, None, None) == -1
    assert L.dfs_sparse_attn_fwd_ex(ctypes.byref(sh), fake, fake, fake, fake, fake, 4, 0.0, ctypes.byref(opts),
                                    odd, None, None) == -3
    assert L.dfs_attn_order(ctypes.byref(sh), None, 4, fake, None) == -1
    assert L.dfs_attn_order(ctypes.byref(sh), fake, 0, fake, None) == -1
    prm = lib.select_params("lvsa", lvsa_T_per=0, lvsa_C=4)
    assert L.dfs_sparse_attn_lvsa_fwd(ctypes.byref(sh), fake, fake, fake, fake, fake, 4, 0.0, ctypes.byref(prm),
                                      fake, None, None) == -1
    prm = lib.select_params("lvsa", lvsa_T_per=2, lvsa_C=4)
    small_frames = _shape_c(lib, H=4, W=8)             # H * W = 32 < blk = 64
    assert L.dfs_sparse_attn_lvsa_fwd(ctypes.byref(small_frames), fake, fake, fake, fake, fake, 4, 0.0,
                                      ctypes.byref(prm), fake, None, None) == -2
    need = lib.dfs_workspace_bytes(lib.Shape(1, 2, 64, 8, 16, 16, 128, 16), lib.DFS_WS_ATTN_BWD)
    assert need > 0
    args = [fake] * 8
    assert L.dfs_sparse_attn_bwd(ctypes.byref(sh), *args, 4, 0.0, fake, fake, fake, fake, 1 << 30, None) == -2
    assert L.dfs_sparse_attn_bwd(ctypes.byref(sh128), *args, 4, 0.0, fake, fake, fake, fake, need - 1, None) == -6
    assert L.dfs_sparse_attn_bwd(ctypes.byref(sh128), *args[:5], None, *args[6:], 4, 0.0, fake, fake, fake, fake,
                                 need, None) == -1
    assert L.dfs_sparse_attn_bwd(ctypes.byref(sh128), *args, 4, 0.0, fake, fake, fake, P((1 << 20) + 16), need,
                                 None) == -3
    prm = lib.select_params("radial", radial_w0=-1)
    assert L.dfs_select_mask(ctypes.byref(sh), None, ctypes.byref(prm), fake, fake, 8, None) == -1
    prm = lib.select_params("radial", radial_w0=8, radial_lambda=-0.5)
    assert L.dfs_select_mask(ctypes.byref(sh), None, ctypes.byref(prm), fake, fake, 8, None) == -1
    big = _shape_c(lib, B=8, nh=16, T=64, H=64, W=64, blk=128, sb=32)   # pooled means >> 32 MiB
    assert L.dfs_block_score_noalloc(ctypes.byref(big), fake, fake, 0.0, fake, None) == -6


def test_noalloc_limit_matches_the_header(lib):
    """The binding's copy of the built-in scratch size is the header's."""
    txt = open(HEADER).read()
    m = re.search(r"#define\s+DFS_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", txt)
    assert m, "DFS_NOALLOC_SCRATCH_BYTES not found"
    assert lib.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


def test_binding_rejects_host_tensors_before_calling_c(lib):
    """The wrappers check tensor arguments on the host: a CPU tensor or a
    missing required tensor raises DfsError(DFS_ERR_INVALID_ARG) without
    reaching the library (so no device pointer is ever formed from it)."""
    import torch
    s = lib.Shape(1, 2, 64, 8, 16, 16, 64, 16)
    x = torch.zeros((1, s.N, 2, 64), dtype=torch.bfloat16)
    scores = torch.zeros((1, 2, s.nb, s.nb), dtype=torch.float32)
    idx = torch.zeros((1, 2, s.nb, 8), dtype=torch.int32)
    cnt = torch.zeros((1, 2, s.nb), dtype=torch.int32)
    calls = [
        lambda: lib.dfs_block_score(s, x, x, 0.0, scores, None),
        lambda: lib.dfs_block_score_noalloc(s, x, x, 0.0, scores),
        lambda: lib.dfs_select_mask(s, scores, lib.select_params("topk", k=8), idx, cnt, 8),
        lambda: lib.dfs_sparse_attn_fwd(s, x, x, x, idx, cnt, 8, 0.0, x),
        lambda: lib.dfs_unperm(s, None, x, x),
        lambda: lib.dfs_attn_order(s, cnt, 8, cnt),
    ]
    for call in calls:
        with pytest.raises(lib.DfsError) as e:
            call()
        assert e.value.status == lib.DFS_ERR_INVALID_ARG
