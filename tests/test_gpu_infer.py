"""Inference side ([PermLLM] "Effect on inference acceleration"): the 2:4
compressed weight, the input-channel gather and the sparse product on the GPU
against the oracle.

Packing and the gather move stored values without arithmetic, so they are
compared bit for bit.  The product accumulates float32 products of the stored
values in an order of its own; each output is checked against the float64
oracle within 1e-5 of the sum of the magnitudes of its terms (float32
accumulation over at most C_in / 2 terms stays well inside that bound).
"""
import numpy as np
import pytest
import torch

from learnable_channel_permutation_b200 import binding as b
from learnable_channel_permutation_b200 import synth
from oracle import lcp_oracle as O

pytestmark = pytest.mark.gpu

TOL_TERMS = 1e-5


def _tdt(dtype):
    return torch.float32 if dtype == "f32" else torch.bfloat16


def _case(cout, cin, B, dtype, seed, outliers=False):
    """Seeded W (values as stored in `dtype`), per-block permutations and the
    2:4 mask of W' = W P_B (the oracle's mask)."""
    rng = np.random.default_rng(seed)
    W = rng.normal(0, 0.02, (cout, cin))
    if outliers:
        W[:, rng.choice(cin, max(1, cin // 100), replace=False)] *= 10
    W = torch.from_numpy(W).to(_tdt(dtype)).float().numpy().astype(np.float64)
    perm = np.stack([rng.permutation(B) for _ in range(cin // B)])
    Wp = O.permute_weight(W, O.perm_matrix(perm))
    M = O.nm_mask(Wp, 2, 4)
    return W, perm, Wp, M


def _dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda().to(_tdt(dtype)).contiguous()


def _pack_gpu(W, perm, M, B, dtype):
    Wd = _dev(W, dtype)
    pd = None if perm is None else torch.from_numpy(np.ascontiguousarray(perm, np.int32)).cuda()
    bits = torch.from_numpy(O.pack_mask_bits(M).view(np.int32)).cuda()
    vals, meta = b.pack24(Wd, pd, bits, B)
    torch.cuda.synchronize()
    return vals, meta, pd


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("cout,cin,B", [(40, 128, 32), (70, 512, 64), (33, 1024, 256), (16, 256, 128)])
def test_pack24_matches_the_oracle_bit_for_bit(gpu_lib, dtype, cout, cin, B):
    W, perm, Wp, M = _case(cout, cin, B, dtype, seed=cout + cin + B)
    vals, meta, _ = _pack_gpu(W, perm, M, B, dtype)
    rv, ri = O.pack_24(Wp, M)
    assert np.array_equal(vals.float().cpu().numpy().astype(np.float64), rv)
    assert np.array_equal(meta.cpu().numpy().view(np.uint32), O.meta_words(ri))
    assert b.device_error() == 0


def test_pack24_without_permutation(gpu_lib):
    rng = np.random.default_rng(5)
    W = torch.from_numpy(rng.normal(size=(24, 256))).to(torch.bfloat16).float().numpy().astype(np.float64)
    M = O.nm_mask(W, 2, 4)
    vals, meta, _ = _pack_gpu(W, None, M, 32, "bf16")
    rv, ri = O.pack_24(W, M)
    assert np.array_equal(vals.float().cpu().numpy().astype(np.float64), rv)
    assert np.array_equal(meta.cpu().numpy().view(np.uint32), O.meta_words(ri))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("T,cin,B", [(1, 256, 32), (7, 512, 64), (130, 4096, 64), (5, 8192, 256), (3, 6144, 128)])
def test_gather_matches_the_oracle_bit_for_bit(gpu_lib, dtype, T, cin, B):
    rng = np.random.default_rng(T + cin)
    X = torch.from_numpy(rng.normal(size=(T, cin))).to(_tdt(dtype))
    perm = np.stack([rng.permutation(B) for _ in range(cin // B)])
    Xd = X.cuda()
    Xp = b.gather(Xd, torch.from_numpy(perm.astype(np.int32)).cuda())
    torch.cuda.synchronize()
    ref = O.gather_channels(X.float().numpy().astype(np.float64), perm)
    assert np.array_equal(Xp.float().cpu().numpy().astype(np.float64), ref)
    assert b.device_error() == 0


def _check_product(Y, vals_np, idx, X64, perm):
    ref = O.sparse24_mm(vals_np, idx, X64, perm)
    bound = O.sparse24_mm(np.abs(vals_np), idx, np.abs(X64), perm)
    err = np.abs(Y - ref)
    assert np.all(err <= TOL_TERMS * bound + 1e-30), float(np.max(err / (bound + 1e-30)))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("T", [1, 2, 3, 8, 16, 37])
@pytest.mark.parametrize("fused", [True, False])
def test_sparse24_mm_matches_the_oracle(gpu_lib, dtype, T, fused):
    cout, cin, B = 200, 1024, 64
    W, perm, Wp, M = _case(cout, cin, B, dtype, seed=T + 7 * fused, outliers=True)
    vals, meta, pd = _pack_gpu(W, perm, M, B, dtype)
    rng = np.random.default_rng(100 + T)
    X = torch.from_numpy(rng.normal(size=(T, cin))).to(_tdt(dtype))
    X64 = X.float().numpy().astype(np.float64)
    if fused:
        Y = b.sparse24_mm(vals, meta, X.cuda(), pd, B)
        Xin, pin = X64, perm
    else:
        Xp = b.gather(X.cuda(), pd)
        Y = b.sparse24_mm(vals, meta, Xp, None, B)
        Xin, pin = X64, perm
    torch.cuda.synchronize()
    rv, ri = O.pack_24(Wp, M)
    _check_product(Y.cpu().numpy().astype(np.float64), rv, ri, Xin, pin)
    assert b.device_error() == 0


@pytest.mark.parametrize("T", [1, 5, 16])
def test_sparse24_mm_cuda_core_path(gpu_lib, T):
    """bf16 with C_in not a multiple of 256 takes the CUDA-core kernel at every
    token count (the other cases cover it at one token and the sparse
    tensor-core kernel from 2 tokens on)."""
    cout, cin, B = 72, 1120, 32
    W, perm, Wp, M = _case(cout, cin, B, "bf16", seed=40 + T)
    vals, meta, pd = _pack_gpu(W, perm, M, B, "bf16")
    rng = np.random.default_rng(41 + T)
    X = torch.from_numpy(rng.normal(size=(T, cin))).to(torch.bfloat16)
    Y = b.sparse24_mm(vals, meta, X.cuda(), pd, B)
    torch.cuda.synchronize()
    rv, ri = O.pack_24(Wp, M)
    _check_product(Y.cpu().numpy().astype(np.float64), rv, ri, X.float().numpy().astype(np.float64), perm)
    assert b.device_error() == 0


@pytest.mark.parametrize("B,T", [(32, 4), (256, 4), (32, 12), (256, 12)])
def test_sparse24_mm_block_sizes_and_wide_rows(gpu_lib, B, T):
    cout, cin = 48, 8192
    W, perm, Wp, M = _case(cout, cin, B, "bf16", seed=B)
    vals, meta, pd = _pack_gpu(W, perm, M, B, "bf16")
    rng = np.random.default_rng(B + 1)
    X = torch.from_numpy(rng.normal(size=(T, cin))).to(torch.bfloat16)
    Y = b.sparse24_mm(vals, meta, X.cuda(), pd, B)
    torch.cuda.synchronize()
    rv, ri = O.pack_24(Wp, M)
    _check_product(Y.cpu().numpy().astype(np.float64), rv, ri, X.float().numpy().astype(np.float64), perm)


@pytest.mark.parametrize("T", [1, 8, 16, 40])
def test_sparse24_mm_full_size_q_proj(gpu_lib, T):
    """The 4096 x 4096 layer of the calibration workload (outlier channels,
    bf16), decode-sized token counts, every output against the oracle."""
    wl = synth.q_proj_4096()
    li = synth.make_inputs(wl)[0]
    W = torch.from_numpy(li.W).to(torch.bfloat16).float().numpy().astype(np.float64)
    rng = np.random.default_rng(9)
    perm = np.stack([rng.permutation(64) for _ in range(4096 // 64)])
    Wp = O.permute_weight(W, O.perm_matrix(perm))
    M = O.nm_mask(Wp, 2, 4)
    vals, meta, pd = _pack_gpu(W, perm, M, 64, "bf16")
    X = torch.from_numpy(li.X[:T]).to(torch.bfloat16)
    Y = b.sparse24_mm(vals, meta, X.cuda(), pd, 64)
    torch.cuda.synchronize()
    rv, ri = O.pack_24(Wp, M)
    _check_product(Y.cpu().numpy().astype(np.float64), rv, ri, X.float().numpy().astype(np.float64), perm)
    assert b.device_error() == 0


def test_deployed_product_equals_the_hardened_training_output(gpu_lib):
    """A hardened GPU step's permutation and mask, packed and applied to the
    calibration tokens, give the oracle's hardened sparse output Y_s."""
    wl = synth.custom(96, 256, 64, 64, 2, 4, 0.5, 5, "bf16", seed=31, outliers=True)
    li = synth.make_inputs(wl)[0]
    W, X, L = (t for t in (torch.from_numpy(li.W).cuda().to(torch.bfloat16),
                           torch.from_numpy(li.X).cuda().to(torch.bfloat16), torch.from_numpy(li.L).cuda()))
    d = b.alloc_outputs(W, X, L, with_mask=True)
    d["perm"] = torch.empty(256 // 64, 64, dtype=torch.int32, device="cuda")
    s = b.Step([d], 64, 2, 4, wl.iters, wl.tau, flags=b.FLAG_HARD)
    s.run()
    vals, meta = b.pack24(W, d["perm"], d["mask"], 64)
    Y = b.sparse24_mm(vals, meta, X, d["perm"], 64)
    torch.cuda.synchronize()
    perm = d["perm"].cpu().numpy().astype(np.int64)
    M = O.unpack_mask_bits(d["mask"].cpu().numpy().view(np.uint32), 256)
    W64 = W.float().cpu().numpy().astype(np.float64)
    X64 = X.float().cpu().numpy().astype(np.float64)
    fw = O.forward(W64, X64, None, 1.0, 5, 2, 4, P=O.perm_matrix(perm), mask=M)
    ref = fw["Ys"].T
    bound = np.abs(fw["A"]) @ np.abs(fw["Xp"])
    assert np.all(np.abs(Y.cpu().numpy() - ref) <= TOL_TERMS * bound.T + 1e-30)
    assert b.device_error() == 0


def test_invalid_groups_and_permutations_are_reported(gpu_lib):
    """A group with three kept bits is written as zeros and reported (301); a
    permutation entry outside [0, B) is skipped and reported (302)."""
    W, perm, Wp, M = _case(8, 128, 32, "bf16", seed=3)
    M = M.copy()
    M[2, 4:8] = [True, True, True, False]
    vals, meta, _ = _pack_gpu(W, perm, M, 32, "bf16")
    assert b.device_error() == 301
    v = vals.float().cpu().numpy()
    assert v[2, 2] == 0 and v[2, 3] == 0
    assert (int(meta.cpu().numpy().view(np.uint32)[2, 0]) >> 4) & 0xF == (0 | 1 << 2)
    bad = torch.from_numpy(perm.astype(np.int32)).cuda()
    bad[1, 5] = 32
    X = torch.zeros(2, 128, dtype=torch.bfloat16, device="cuda")
    b.gather(X, bad)
    torch.cuda.synchronize()
    assert b.device_error() == 302
    b.sparse24_mm(vals, meta, X, bad, 32)
    torch.cuda.synchronize()
    assert b.device_error() == 302
    assert b.device_error() == 0
