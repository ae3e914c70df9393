"""The C-ABI library loads, exports every entry point the header declares, and
rejects bad arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z][a-z0-9_]*)\s*\(", src)) - {"sizeof"})


def test_header_parses_to_entry_points():
    names = _declared()
    for must in ["moe_route", "moe_permute", "fp8_quant_1x128", "fp8_grouped_gemm_blockscaled",
                 "swiglu_requant", "moe_combine", "moe_bias_update"]:
        assert must in names


def test_library_exports_every_declared_symbol():
    from sparse_moe_layer_group_b200 import _abi
    lib = ctypes.CDLL(_abi.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(_declared()) == set(_abi.EXPORTED)


def test_status_strings_and_version():
    from sparse_moe_layer_group_b200 import _abi
    assert _abi.status_string(0) == "MOE_OK"
    assert "INVALID_ARG" in _abi.status_string(1)
    assert "unknown" in _abi.status_string(99)
    assert _abi.abi_version() >= 1


def test_workspace_size_scales_with_tokens():
    from sparse_moe_layer_group_b200 import _abi
    small = _abi.workspace_size(_abi.dims(64, 256, 16, 4, 4, 2, 128, 2.5))
    big = _abi.workspace_size(_abi.dims(4096, 7168, 256, 8, 8, 4, 2048, 2.5))
    assert big >= 4096 * 256 * 4 and small > 0 and small % 256 == 0


def test_host_validation_rejects_before_launch():
    from sparse_moe_layer_group_b200 import _abi as a
    L = a._lib
    # cols not a multiple of 128
    assert L.fp8_quant_1x128(16, 4, 100, 16, 16, None, None) == a.MOE_ERR_INVALID_ARG
    # NULL pointers
    assert L.fp8_quant_1x128(None, 4, 128, None, None, None, None) == a.MOE_ERR_INVALID_ARG
    # misaligned pointer
    assert L.fp8_quant_1x128(18, 4, 128, 16, 16, None, None) == a.MOE_ERR_INVALID_ARG
    # E not divisible by n_group; topk_group * group size < K; K too large
    for d in [a.dims(8, 256, 16, 4, 3, 2, 128, 2.5), a.dims(8, 256, 16, 5, 4, 1, 128, 2.5),
              a.dims(8, 256, 2048, 4, 4, 2, 128, 2.5)]:
        rc = L.moe_route(ctypes.byref(d), 16, 16, 16, None, 16, 16, None, None, 0, None, None)
        assert rc in (a.MOE_ERR_INVALID_ARG, a.MOE_ERR_UNSUPPORTED)
    # workspace missing
    d = a.dims(8, 256, 16, 4, 4, 2, 128, 2.5)
    assert L.moe_route(ctypes.byref(d), 16, 16, 16, None, 16, 16, None, None, 0, None, None) == a.MOE_ERR_WORKSPACE
    assert L.moe_permute(ctypes.byref(d), 16, None, None, 16, 16, 16, 16, None, None, 16, 8, None,
                         None) == a.MOE_ERR_WORKSPACE
    # GEMM: K not a multiple of 128, bad epilogue, SwiGLU without scale output
    assert L.fp8_grouped_gemm_blockscaled(1, 16, 64, 256, 100, 16, 16, 16, 16, 0, 16, None, None,
                                          None) == a.MOE_ERR_INVALID_ARG
    assert L.fp8_grouped_gemm_blockscaled(1, 16, 64, 256, 128, 16, 16, 16, 16, 9, 16, None, None,
                                          None) == a.MOE_ERR_INVALID_ARG
    assert L.fp8_grouped_gemm_blockscaled(1, 16, 64, 256, 128, 16, 16, 16, 16, 2, 16, None, None,
                                          None) == a.MOE_ERR_INVALID_ARG
    # more groups than the kernel's shared-memory group table holds (limit 4000, both tile modes)
    for mode in (0, a.MOE_GEMM_PAIR_CTA):
        assert L.fp8_grouped_gemm_blockscaled(4001, 16, 64, 256, 128, 16, 16, 16, 16, mode, 16, None, None,
                                              None) == a.MOE_ERR_UNSUPPORTED
    # gather variant: the row map is required and 4-byte aligned, a_rows >= 1
    gg = L.fp8_grouped_gemm_blockscaled_gather
    assert gg(1, 16, 64, 256, 128, 16, 16, 8, None, 16, 16, 0, 16, None, None, None) == a.MOE_ERR_INVALID_ARG
    assert gg(1, 16, 64, 256, 128, 16, 16, 8, 18, 16, 16, 0, 16, None, None, None) == a.MOE_ERR_INVALID_ARG
    assert gg(1, 16, 64, 256, 128, 16, 16, -1, 16, 16, 16, 0, 16, None, None, None) == a.MOE_ERR_INVALID_ARG
    assert gg(1, 16, 64, 256, 128, 16, 16, 0, 16, 16, 16, 0, 16, None, None, None) == a.MOE_ERR_INVALID_ARG
    assert gg(1, 16, 64, 256, 100, 16, 16, 8, 16, 16, 16, 0, 16, None, None, None) == a.MOE_ERR_INVALID_ARG
    assert gg(0, 16, 64, 256, 128, 16, 16, 8, 16, 16, 16, 0, 16, None, None, None) == 0
    # combine variant: token and gate maps required and 4-byte aligned, out_rows >= 1; finish n % 8 == 0
    gc = L.fp8_grouped_gemm_blockscaled_combine
    assert gc(1, 16, 64, 256, 128, 16, 16, 16, 16, None, 16, 8, 16, None, None) == a.MOE_ERR_INVALID_ARG
    assert gc(1, 16, 64, 256, 128, 16, 16, 16, 16, 16, 18, 8, 16, None, None) == a.MOE_ERR_INVALID_ARG
    assert gc(1, 16, 64, 256, 128, 16, 16, 16, 16, 16, 16, 0, 16, None, None) == a.MOE_ERR_INVALID_ARG
    assert gc(0, 16, 64, 256, 128, 16, 16, 16, 16, 16, 16, 8, 16, None, None) == 0
    assert L.moe_combine_finish(16, 12, 16, None, 1, None) == a.MOE_ERR_INVALID_ARG
    assert L.moe_combine_finish(16, 0, 16, None, 1, None) == 0
    # one-call forward and host runner: the struct and buffers are required, n >= 0
    assert L.moe_layer_forward(None, 16, 16, None) == a.MOE_ERR_INVALID_ARG
    lay = a.MoeLayerC()
    assert L.moe_layer_forward(ctypes.byref(lay), None, 16, None) == a.MOE_ERR_INVALID_ARG
    assert L.moe_layer_run_host(ctypes.byref(lay), None, None, -1, None, None, None) == a.MOE_ERR_INVALID_ARG
    assert L.moe_layer_run_host(ctypes.byref(lay), None, None, 0, None, None, None) == 0
    # zero-size work is a no-op
    assert L.fp8_grouped_gemm_blockscaled(0, 16, 64, 256, 128, 16, 16, 16, 16, 0, 16, None, None, None) == 0
    assert L.fp8_quant_1x128(16, 0, 128, 16, 16, None, None) == 0
    assert L.swiglu_requant(16, 4, 100, 16, 16, None, None) == a.MOE_ERR_INVALID_ARG
    assert L.moe_bias_update(0, 4, 2, 0.001, 16, 16, None) == a.MOE_ERR_INVALID_ARG
    assert L.moe_combine(None, 16, 16, 16, None, 16, None, None) == a.MOE_ERR_INVALID_ARG


def test_wgrad_host_validation():
    from sparse_moe_layer_group_b200 import _abi as a
    L = a._lib
    # columns not a multiple of 128, padded capacity not a multiple of 16
    assert L.fp8_quant_128x1_grouped(16, 4, 100, 1, 16, 16, 128, 16, 2, None, None) == a.MOE_ERR_INVALID_ARG
    assert L.fp8_quant_128x1_grouped(16, 4, 128, 1, 16, 16, 130, 16, 2, None, None) == a.MOE_ERR_INVALID_ARG
    # too many groups; no groups is a no-op
    assert L.fp8_quant_128x1_grouped(16, 4, 128, 5000, 16, 16, 128, 16, 2, None, None) == a.MOE_ERR_UNSUPPORTED
    assert L.fp8_grouped_gemm_wgrad(0, None, 0, 128, 128, None, None, None, None, 0, 0, None, None, None) == a.MOE_OK
    assert L.fp8_grouped_gemm_wgrad(2, 16, 4, 100, 128, 16, 16, 16, 16, 128, 2, 16, None, None) == \
        a.MOE_ERR_INVALID_ARG
    assert L.fp8_grouped_gemm_wgrad(5000, 16, 4, 128, 128, 16, 16, 16, 16, 128, 2, 16, None, None) == \
        a.MOE_ERR_UNSUPPORTED
    # NULL operands
    assert L.fp8_grouped_gemm_wgrad(2, 16, 4, 128, 128, None, 16, 16, 16, 128, 2, 16, None, None) == \
        a.MOE_ERR_INVALID_ARG


def test_python_bindings_marshal_zero_size_calls():
    """The Python binding of each expert-parallel call passes the argument count
    and types the C entry point declares (zero-size calls return before any
    device work, so this runs without a GPU)."""
    import torch
    from sparse_moe_layer_group_b200 import _abi as a
    i32, f32 = torch.int32, torch.float32
    idx, w = torch.empty(0, 8, dtype=i32), torch.empty(0, 8, dtype=f32)
    a.moe_ep_plan(idx, w, 16, 2, a.MOE_EP_BLOCK, torch.empty(0, dtype=i32), torch.empty(0, 8, dtype=i32),
                  torch.empty(0, 8, dtype=f32), None, 0)
    a.moe_ep_scatter_rows(torch.empty(0, dtype=i32), torch.empty(0, 4, dtype=i32), torch.empty(0, 4, dtype=i32), 0)
    a.moe_ep_split(torch.empty(0, 8, dtype=i32), 16, 2, torch.empty(0, dtype=i32), torch.empty(0, dtype=i32), None, 0)
    a.moe_ep_scatter(torch.empty(0, dtype=i32), torch.empty(0, dtype=i32), torch.empty(0, dtype=i32), 0)
    with pytest.raises(a.MoEError):
        a.moe_ep_plan(torch.empty(2, 8, dtype=i32), torch.empty(2, 8, dtype=f32), 16, 3, a.MOE_EP_BLOCK,
                      torch.empty(16, dtype=i32), torch.empty(16, 8, dtype=i32), torch.empty(16, 8, dtype=f32),
                      None, 0)                            # 16 experts do not divide over 3 ranks


def test_layer_struct_layout_matches_the_header(tmp_path):
    """The ctypes mirror of moe_layer has the header's size and field offsets
    (a C program built from the header prints them)."""
    import shutil
    import subprocess
    from sparse_moe_layer_group_b200 import _abi as a
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    fields = [f for f, _ in a.MoeLayerC._fields_]
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "moe_b200.h"\nint main(void) {\n'
                   '  printf("%zu\\n", sizeof(moe_layer));\n' +
                   "".join(f'  printf("%zu\\n", offsetof(moe_layer, {f}));\n' for f in fields) + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()]
    want = [ctypes.sizeof(a.MoeLayerC)] + [getattr(a.MoeLayerC, f).offset for f in fields]
    assert got == want
