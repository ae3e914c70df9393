"""moe_permute_noalloc: the permutation for callers that cannot allocate device
memory (its scratch is a static array inside the library), checked against
moe_permute with a caller workspace on the same inputs, through the C ABI.

This file is named so that pytest collects it last."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _buffers(T, E, K, H):
    dev = dict(device="cuda")
    return dict(load=torch.full((E,), -1, dtype=torch.int32, **dev),
                offs=torch.full((E + 1,), -1, dtype=torch.int32, **dev),
                tok_of=torch.full((T * K,), -1, dtype=torch.int32, **dev),
                row_of=torch.full((T * K,), -1, dtype=torch.int32, **dev),
                aq=torch.zeros(T * K, H, dtype=torch.uint8, **dev),
                as_=torch.zeros(T * K, H // 128, dtype=torch.float32, **dev),
                st=torch.zeros(1, dtype=torch.int32, **dev))


def _run_pair(lib, T, E, K, H, seed, skew):
    idx = synth.topk_indices(T, E, K, seed, skew=skew).cuda()
    x = synth.activations(T, H, seed + 1, device="cuda")
    xq = torch.empty(T, H, dtype=torch.uint8, device="cuda")
    xs = torch.empty(T, H // 128, dtype=torch.float32, device="cuda")
    lib.fp8_quant_1x128(x, xq, xs)
    d = lib.dims(T, H, E, K, 1, 1, 128, 2.5)
    ref = _buffers(T, E, K, H)
    ws = torch.empty(lib.workspace_size(d), dtype=torch.uint8, device="cuda")
    lib.moe_permute(d, idx, xq, xs, ref["load"], ref["offs"], ref["tok_of"], ref["row_of"], ref["aq"],
                    ref["as_"], ws, ref["st"])
    got = _buffers(T, E, K, H)
    lib.abi.moe_permute_noalloc(d, idx, xq, xs, got["load"], got["offs"], got["tok_of"], got["row_of"],
                                got["aq"], got["as_"], got["st"])
    torch.cuda.synchronize()
    for k in ref:
        assert torch.equal(ref[k], got[k]), k


def test_noalloc_matches_workspace_call_twice(lib):
    # first call: a large, skewed batch; second call: a smaller one, so the
    # static scratch still holds the first call's counts when it starts
    _run_pair(lib, T=4096, E=256, K=8, H=512, seed=21, skew=4.0)
    _run_pair(lib, T=300, E=32, K=4, H=256, seed=22, skew=0.0)


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    cap = lib.abi.moe_permute_noalloc_max_scratch()
    assert cap == 1 << 20
    E = 256
    T = (cap // (4 * E)) * 32 + 1            # one 32-token chunk too many
    d = lib.dims(T, 128, E, 8, 1, 1, 128, 2.5)
    with pytest.raises(lib.MoEError) as ei:
        lib.abi.moe_permute_noalloc(d, None, None, None, None, None, None, None, None, None)
    assert ei.value.code in (lib.abi.MOE_ERR_TOO_LARGE, lib.abi.MOE_ERR_INVALID_ARG)
    # with valid output pointers the size check is what rejects it
    load = torch.empty(E, dtype=torch.int32, device="cuda")
    offs = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    with pytest.raises(lib.MoEError) as ei:
        lib.abi.moe_permute_noalloc(d, None, None, None, load, offs, None, None, None, None)
    assert ei.value.code == lib.abi.MOE_ERR_TOO_LARGE
