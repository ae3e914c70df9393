"""GPU parity of the gather variant of the grouped FP8 GEMM: GEMM row m reads
A row a_map[m] (and its scales) of a source matrix instead of a permuted copy.

The rows are fetched by TMA row gathers (four rows per instruction).  Each case
is checked two ways: bit for bit against the plain grouped GEMM run
on the materialised copy A[a_map] (same codes and scales in the same tensor-core
tiles, so every epilogue must give the same bits), and against the float64
oracle on that copy.  Maps repeat rows and leave some unused, as the layer's
routing does; rows outside every group are never written."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._util import TOL_NORMWISE, cuda, normwise, np_

pytestmark = pytest.mark.gpu

GATHER_CASES = [  # group sizes, N, K, source rows
    ([200], 512, 1024, 64),                        # one group, ragged M tile, ring wraps
    ([0, 130, 1, 257, 40], 512, 256, 97),          # empty and 1-row groups
    ([5] * 40, 256, 384, 33),                      # many small groups
    (list(range(0, 300, 7)), 768, 512, 300),       # > 148 tiles: persistent loop
    ([90, 3, 300, 2100], 512, 256, 700),           # large last group: its tiles run in two chunks
]


def _case(sizes, N, K, R, seed):
    G = len(sizes)
    M = int(sum(sizes)) + 5                     # 5 rows outside every group
    x = synth.heavy_tailed(R, K, seed)
    b = synth.normal((G * N, K), 0.02, seed + 1, dtype=torch.bfloat16).reshape(G, N, K)
    rng = np.random.default_rng(seed)
    amap = rng.integers(0, R, M).astype(np.int32)
    amap[-5:] = -7                              # never read: outside every group
    offs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    return x, b, amap, offs, M


def _quantised(lib, x, b):
    R, K = x.shape
    G, N, _ = b.shape
    qx = torch.empty(R, K, dtype=torch.uint8, device="cuda")
    sx = torch.empty(R, K // 128, dtype=torch.float32, device="cuda")
    lib.fp8_quant_1x128(cuda(x), qx, sx)
    qb = torch.empty(G, N, K, dtype=torch.uint8, device="cuda")
    sb = torch.empty(G, N // 128, K // 128, dtype=torch.float32, device="cuda")
    lib.fp8_quant_128x128(cuda(b), qb, sb)
    return qx, sx, qb, sb


def _run(lib, gather, G, goffs, M, N, K, qa, sa, gmap, qb, sb, epi):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if epi == "swiglu":
        C = torch.full((M, N // 2), 0x55, dtype=torch.uint8, device="cuda")
        sC = torch.full((M, N // 256), -1.0, dtype=torch.float32, device="cuda")
        e = lib.MOE_EPI_SWIGLU_REQUANT
    else:
        C = torch.full((M, N), 7.0, dtype=torch.float32 if epi == "f32" else torch.bfloat16, device="cuda")
        sC = None
        e = lib.MOE_EPI_F32 if epi == "f32" else lib.MOE_EPI_BF16
    if gather:
        lib.fp8_grouped_gemm_blockscaled_gather(G, goffs, M, N, K, qa, sa, gmap, qb, sb, e, C, sC, st)
    else:
        lib.fp8_grouped_gemm_blockscaled(G, goffs, M, N, K, qa, sa, qb, sb, e | 0x100, C, sC, st)
    torch.cuda.synchronize()
    return C, sC, int(st.item())


@pytest.mark.parametrize("sizes,N,K,R", GATHER_CASES)
@pytest.mark.parametrize("epi", ["f32", "bf16", "swiglu"])
def test_gather_gemm(lib, sizes, N, K, R, epi):
    if epi == "swiglu" and N % 256:
        N += 128
    x, b, amap, offs, M = _case(sizes, N, K, R, seed=len(sizes) * 5 + N + K + R)
    qx, sx, qb, sb = _quantised(lib, x, b)
    G, used = len(sizes), int(offs[-1])
    goffs, gmap = cuda(torch.from_numpy(offs)), cuda(torch.from_numpy(amap))
    # the materialised copy the plain GEMM reads (rows outside every group: row 0)
    idx = torch.from_numpy(np.where(amap >= 0, amap, 0).astype(np.int64)).cuda()
    qa, sa = qx[idx].contiguous(), sx[idx].contiguous()
    Cg, sCg, stg = _run(lib, True, G, goffs, M, N, K, qx, sx, gmap, qb, sb, epi)
    Cm, sCm, stm = _run(lib, False, G, goffs, M, N, K, qa, sa, gmap, qb, sb, epi)
    assert stg == 0 and stm == 0
    assert torch.equal(Cg[:used], Cm[:used])
    if epi == "swiglu":
        assert torch.equal(sCg[:used], sCm[:used])
        assert bool((Cg[used:] == 0x55).all()) and bool((sCg[used:] == -1.0).all())
    else:
        assert bool((Cg[used:] == 7.0).all())
        # and against the oracle on the same copy
        xq, xs = oracle.quant_1x128(x.float().numpy())
        bq = np.stack([oracle.quant_128x128(b[g].float().numpy())[0] for g in range(G)])
        bs = np.stack([oracle.quant_128x128(b[g].float().numpy())[1] for g in range(G)])
        rm = np.where(amap >= 0, amap, 0)
        ref = oracle.grouped_gemm_blockscaled(offs, xq[rm], xs[rm], bq, bs)[:used]
        if epi == "bf16":
            ref = oracle.round_bf16(ref)
        assert normwise(np_(Cg)[:used].astype(np.float64), ref) < TOL_NORMWISE


def test_gather_layer_map(lib):
    """The layer's map: routed rows through tok_of, then 0..T-1 for the shared
    expert's group (every source row read K + 1 times)."""
    T, K, E, H, N = 300, 4, 6, 512, 512
    rng = np.random.default_rng(3)
    tok = np.concatenate([np.sort(rng.choice(T, K * T // E, replace=True)) for _ in range(E)]).astype(np.int32)
    sizes = [len(tok) // E] * E + [T]
    amap = np.concatenate([tok, np.arange(T, dtype=np.int32)])
    x = synth.activations(T, H, 4)
    b = synth.normal(((E + 1) * N, H), 0.02, 5, dtype=torch.bfloat16).reshape(E + 1, N, H)
    qx, sx, qb, sb = _quantised(lib, x, b)
    offs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    M = int(offs[-1])
    goffs, gmap = cuda(torch.from_numpy(offs)), cuda(torch.from_numpy(amap))
    idx = torch.from_numpy(amap.astype(np.int64)).cuda()
    Cg, sCg, stg = _run(lib, True, E + 1, goffs, M, N, H, qx, sx, gmap, qb, sb, "swiglu")
    Cm, sCm, stm = _run(lib, False, E + 1, goffs, M, N, H, qx[idx].contiguous(), sx[idx].contiguous(), gmap, qb, sb,
                        "swiglu")
    assert stg == 0 and stm == 0
    assert torch.equal(Cg, Cm) and torch.equal(sCg, sCm)


def test_gather_bad_index(lib):
    """A map entry outside [0, a_rows) inside a group raises MOE_FLAG_BAD_INDEX;
    nothing outside A is read, and every other row is unaffected (the flagged
    rows' values are unspecified)."""
    sizes, N, K, R = [40, 100], 256, 256, 50
    x, b, amap, offs, M = _case(sizes, N, K, R, seed=11)
    amap[17] = R                 # one past the end
    amap[60] = -3
    qx, sx, qb, sb = _quantised(lib, x, b)
    goffs, gmap = cuda(torch.from_numpy(offs)), cuda(torch.from_numpy(amap))
    Cg, _, stg = _run(lib, True, len(sizes), goffs, M, N, K, qx, sx, gmap, qb, sb, "f32")
    assert stg & lib.MOE_FLAG_BAD_INDEX
    good = np.where(amap >= 0, np.minimum(amap, R - 1), 0)
    idx = torch.from_numpy(good.astype(np.int64)).cuda()
    Cm, _, stm = _run(lib, False, len(sizes), goffs, M, N, K, qx[idx].contiguous(), sx[idx].contiguous(), gmap,
                      qb, sb, "f32")
    used = int(offs[-1])
    bad = [17, 60]
    ok = np.setdiff1d(np.arange(used), bad)
    assert torch.equal(Cg[ok], Cm[ok])
