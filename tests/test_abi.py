"""The C ABI library: it loads without a GPU, exports every entry point that
include/*.h declares, and rejects bad arguments on the host before any CUDA
call."""
import ctypes
import glob
import os
import re

import pytest

from segmented_fine_tuning_b200 import _binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        txt = open(h).read()
        txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
        for m in re.finditer(r"^\s*(?:HGA_API\s+)?(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s+(hga_[a-z0-9_]+)\s*\(", txt, re.M):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from segmented_fine_tuning_b200 import build
    build.build()
    return _binding.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 11, names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_binding_covers_every_symbol():
    bound = {n for n, _, _ in _binding._SIGNATURES}
    assert set(_declared_functions()) <= bound


def test_status_strings(lib):
    for code, name in _binding.STATUS_NAMES.items():
        assert lib.hga_status_string(code).decode() == name


def _dims(**kw):
    base = dict(B=1, Hq=4, Hkv=2, d=128, block=128, S=256, n_hist_blocks=4, topk=2, dtype=1)
    base.update(kw)
    return _binding.hga_dims(**base)


BAD_DIMS = [
    dict(Hq=3),          # Hq % Hkv
    dict(d=96),          # head dim
    dict(block=48),      # block size
    dict(S=200),         # S % block
    dict(topk=0),        # K >= 1
    dict(topk=65),       # K <= 64
    dict(B=0),
    dict(n_hist_blocks=-1),
    dict(q_block=48),                      # query-block size
    dict(block=32, S=96, q_block=64),      # S % q_block
]


@pytest.mark.parametrize("kw", BAD_DIMS)
def test_bad_shapes_rejected_on_host(lib, kw):
    d = _dims(**kw)
    p = ctypes.c_void_p(16)
    st = lib.hga_attn_fwd(ctypes.byref(d), p, p, p, p, p, 4, p, p, p, None)
    assert st == 2, (kw, st, lib.hga_last_error())
    assert lib.hga_last_error()


def test_null_and_invalid_arguments(lib):
    d = _dims()
    p = ctypes.c_void_p(16)
    assert lib.hga_attn_fwd(None, p, p, p, p, p, 4, p, p, p, None) == 1
    assert lib.hga_attn_fwd(ctypes.byref(d), None, p, p, p, p, 4, p, p, p, None) == 1
    assert lib.hga_attn_fwd(ctypes.byref(d), p, p, p, None, p, 4, p, p, p, None) == 1   # history missing
    assert lib.hga_attn_fwd(ctypes.byref(d), ctypes.c_void_p(18), p, p, p, p, 4, p, p, p, None) == 1  # misaligned
    assert lib.hga_attn_fwd(ctypes.byref(d), p, p, p, p, p, 4, p, ctypes.c_void_p(24), p, None) == 1  # o misaligned
    assert "o must be 16-byte aligned" in lib.hga_last_error().decode()
    assert lib.hga_block_summaries(ctypes.byref(d), p, 0, 9, p, None) == 1   # range past n_hist_blocks
    assert lib.hga_block_summaries(ctypes.byref(d), p, 3, 1, p, None) == 1
    assert lib.hga_select_topk(ctypes.byref(_dims(n_hist_blocks=5000)), p, p, p, None, None) == 2
    # workspace too small
    ws = lib.hga_attn_bwd_workspace_size(ctypes.byref(d))
    assert ws >= 4 * 4 * 256 and ws % 256 == 0
    assert lib.hga_attn_bwd(ctypes.byref(d), p, p, p, p, p, 4, p, p, p, p, p, p, p, ctypes.c_void_p(256), ws - 1,
                            None) == 1
    assert lib.hga_selftest_umma(7, p, p, p, None) == 1
    assert lib.hga_offload_segment(ctypes.byref(d), p, p, p, p, 4, 3, None) == 1  # 2 blocks at 3 > capacity 4


def test_new_entry_points_validate_on_host(lib):
    """Decode, sparse backward, segment append and zero-copy gather reject bad
    arguments before touching a device."""
    d = _dims()
    p = ctypes.c_void_p(16)
    ws = lib.hga_decode_workspace_size(ctypes.byref(d), 1)
    assert ws > 0 and ws % 256 == 0
    assert lib.hga_decode_workspace_size(ctypes.byref(d), 0) == 0       # n_q < 1
    assert lib.hga_decode_workspace_size(ctypes.byref(d), 129) == 0     # n_q > block
    # n_q outside [1, block]
    assert lib.hga_decode_select(ctypes.byref(d), 0, p, p, p, None, p, ws, None) == 2
    assert lib.hga_decode_attn(ctypes.byref(d), 200, 0, p, p, p, p, p, 4, p, p, p, p, ws, None) == 2
    # new tokens past the segment buffer (S = 256)
    assert lib.hga_decode_attn(ctypes.byref(d), 2, 255, p, p, p, p, p, 4, p, p, p, p, ws, None) == 2
    # short workspace
    assert lib.hga_decode_select(ctypes.byref(d), 1, p, p, p, None, p, 8, None) == 1
    assert lib.hga_decode_attn(ctypes.byref(d), 1, 0, p, p, p, p, p, 4, p, p, p, p, 8, None) == 1
    # sparse backward: mask required, scale finite
    wsb = lib.hga_attn_bwd_workspace_size(ctypes.byref(d))
    w256 = ctypes.c_void_p(256)
    assert lib.hga_attn_bwd_sparse(ctypes.byref(d), p, p, p, p, p, 4, p, p, p, p, None, 1.0, p, p, p, w256, wsb,
                                   None) == 1
    assert lib.hga_attn_bwd_sparse(ctypes.byref(d), p, p, p, p, p, 4, p, p, p, p, p, float("inf"), p, p, p, w256,
                                   wsb, None) == 1
    # append: blocks outside the summary array, host tier halves must come together
    assert lib.hga_append_segment(ctypes.byref(d), p, p, 3, p, None, None, None, None, None, 0, None, None) == 1
    assert lib.hga_append_segment(ctypes.byref(d), p, p, 0, p, None, None, None, p, None, 8, None, None) == 1
    # gather: a pool of no slots, a tier shorter than the history
    assert lib.hga_gather_blocks_mapped(ctypes.byref(d), p, p, 4, p, p, p, 0, p, None) == 1
    assert lib.hga_gather_blocks_mapped(ctypes.byref(d), p, p, 3, p, p, p, 4, p, None) == 1


def test_binding_rejects_wrong_shapes():
    import torch
    D = _binding.Dims(1, 4, 2, 128, 128, 256, 4, 2, "bf16")
    q = torch.zeros((1, 256, 4, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        _binding.hga_attn_fwd(D, q, q, q, q, q, 4, q, q, q)


def test_oracle_and_library_share_nothing():
    """The CUDA sources and the oracle neither include nor import each other."""
    csrc = glob.glob(os.path.join(ROOT, "segmented_fine_tuning_b200", "**", "*"), recursive=True)
    for f in csrc:
        if f.endswith((".cu", ".cuh", ".h", ".py")):
            txt = open(f).read()
            assert "oracle" not in re.sub(r"#.*|//.*", "", txt).lower() or f.endswith("build.py"), f
    for f in glob.glob(os.path.join(ROOT, "oracle", "*")):
        if f.endswith((".c", ".h", ".py")):
            assert "segmented_fine_tuning_b200" not in open(f).read(), f


def test_headers_compile_as_c_and_cpp(tmp_path):
    """The boundary is a C ABI: both public headers compile as C11 (no C++
    in the signatures) and as C++17, warning-free, with only the CUDA runtime
    headers on the include path."""
    import shutil
    import subprocess
    cc, cxx = shutil.which("gcc"), shutil.which("g++")
    if not cc or not cxx:
        pytest.skip("no host compiler")
    src = tmp_path / "use.c"
    src.write_text('#include "hga.h"\n#include "hga_selftest.h"\n'
                   "int main(void) { hga_dims d; hga_block_cache c; (void)d; (void)c; return 0; }\n")
    from torch.utils.cpp_extension import CUDA_HOME
    if not CUDA_HOME:
        pytest.skip("no CUDA toolkit headers")
    inc = ["-I" + os.path.join(ROOT, "include"), "-I" + os.path.join(CUDA_HOME, "include")]
    for tool, lang in ((cc, ["-std=c11"]), (cxx, ["-std=c++17", "-x", "c++"])):
        r = subprocess.run([tool, *lang, "-Wall", "-Wextra", "-Werror", *inc, "-c", str(src), "-o",
                            str(tmp_path / "use.o")], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_size_limits_rejected_on_host(lib):
    """One past each documented maximum is rejected with HGA_ERR_SHAPE before
    any device work: 4,096 history blocks for a selection (prefill and
    decode), 128 blocks for an appended segment."""
    p = ctypes.c_void_p(16)
    d = _dims(n_hist_blocks=4097, block=32, S=128)
    assert lib.hga_select_topk(ctypes.byref(d), p, p, p, None, None) == 2
    assert "4096" in lib.hga_last_error().decode()
    ws = ctypes.c_size_t(1 << 30)
    assert lib.hga_decode_select(ctypes.byref(d), 1, p, p, p, None, p, ws, None) == 2
    d = _dims(n_hist_blocks=4096, block=32, S=128)
    assert lib.hga_decode_workspace_size(ctypes.byref(d), 1) > 0
    d = _dims(S=129 * 128, n_hist_blocks=129 * 128 // 128 + 1)
    assert lib.hga_append_segment(ctypes.byref(d), p, p, 0, p, None, None, None, None, None, 0, None, None) == 2
    assert "128" in lib.hga_last_error().decode()


def test_forward_heads_per_cta_setter(lib):
    """Host-only knob: 0, 1 and 2 are accepted, anything else is rejected."""
    for h in (1, 2, 0):
        assert lib.hga_set_forward_heads_per_cta(h) == 0
    for h in (-1, 3):
        assert lib.hga_set_forward_heads_per_cta(h) == 1
        assert "heads per CTA" in lib.hga_last_error().decode()
    assert lib.hga_set_forward_heads_per_cta(0) == 0


@pytest.mark.parametrize("kw,nkv,want", [
    (dict(), 4, 1),                                        # bf16, d128, block 128
    (dict(d=64), 4, 1),                                    # head dim 64
    (dict(block=64, q_block=128), 9, 1),                   # 64-token history blocks, two per tile
    (dict(block=64, q_block=128, n_hist_blocks=40000, topk=4), 40000, 0),  # block indices past 15 bits
    (dict(block=32, q_block=128, n_hist_blocks=40000, topk=4), 40000, 1),  # grouped tiles: no such limit
    (dict(block=32, q_block=128), 4, 1),                   # 32-token history blocks, four per tile
    (dict(block=16, q_block=128), 4, 1),                   # 16-token history blocks, eight per tile
    (dict(block=64), 9, 0),                                # 64-row query blocks: CUDA-core kernels
    (dict(block=128, q_block=64), 4, 0),
    (dict(dtype=0), 4, 0),                                 # fp32
    (dict(Hq=6, Hkv=2), 4, 0),                             # odd group size
    (dict(block=32), 4, 0),                                # 32-row query blocks: CUDA-core kernels
    (dict(q_block=48), 4, -1),                             # rejected dims
])
def test_tensor_core_path_selection(lib, kw, nkv, want):
    """Which kernels the attention calls use for a shape (host-only query)."""
    d = _dims(**kw)
    assert lib.hga_attn_uses_tensor_cores(ctypes.byref(d), nkv) == want, (kw, lib.hga_last_error())
