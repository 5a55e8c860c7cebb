"""Parity of the three tcgen05 GEMMs (lmhead_fwd, lmhead_bwd_dx, lmhead_bwd_dw)
with the FP64 oracle, through the C ABI.

Integer-valued BF16 operands in [-8, 8] make every partial sum exact in FP32
(Megatron-LM PR #6252, "Integer bitwise exactness results"), so those cases
compare raw words; random operands use the K-scaled absolute tolerance."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from lm_head_fp32_b200 import lmhead, synth
from helpers import assert_abs_close, assert_bf16_close, bits, gemm_tol, guarded_empty, guarded_full, logits_tol, to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def status_word():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def gpu_logits(X, W, dtype=torch.float32):
    M, V = X.shape[0], W.shape[0]
    out = guarded_empty((M, V), dtype)
    st = status_word()
    lmhead.lmhead_fwd(X.to(DEV), W.to(DEV), out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return out


def gpu_dx(dl, W, dtype=torch.float32):
    out = guarded_empty((dl.shape[0], W.shape[1]), dtype)
    st = status_word()
    lmhead.lmhead_bwd_dx(dl.to(DEV), W.to(DEV), out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return out


def gpu_dw(dl, X, dtype=torch.float32):
    out = guarded_empty((dl.shape[1], X.shape[1]), dtype)
    st = status_word()
    lmhead.lmhead_bwd_dw(dl.to(DEV), X.to(DEV), out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return out


def test_integer_exactness_k_sweep(golden_dir):
    """16 x K activations, 32768 x K weights, BF16 integers in [-8,8], seed 1234,
    K in {512..16384}: the FP32 logits equal the exact result word for word."""
    spec = json.load(open(os.path.join(golden_dir, "p1_integer_exactness.json")))
    M, V = spec["activations_rows"], spec["vocab_rows"]
    for K in spec["K"]:
        X = synth.int_bf16((M, K), spec["seed"], spec["int_lo"], spec["int_hi"])
        W = synth.int_bf16((V, K), spec["seed"] + 1, spec["int_lo"], spec["int_hi"])
        out = gpu_logits(X, W)
        ref = oracle.round_f32(oracle.logits(bits(X), bits(W)))
        got = out.cpu().numpy()
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), f"K={K}"
        # the BF16 epilogue of the same kernel is the RNE of the same exact value
        out16 = gpu_logits(X, W, torch.bfloat16)
        ref16 = oracle.round_bf16(oracle.logits(bits(X), bits(W)))
        assert np.array_equal(bits(out16), ref16), f"K={K} (BF16 epilogue)"


@pytest.mark.parametrize("M,K,V", [(300, 1000, 1000), (17, 72, 32776), (130, 4096, 520),
                                   (1, 8, 1), (257, 136, 129), (1024, 256, 384),
                                   (64, 520, 4104), (100, 1024, 8200), (100, 16384, 1032)])
def test_logits_random_ragged(M, K, V):
    X = synth.normal_bf16((M, K), 1.0, 11 + M)
    W = synth.normal_bf16((V, K), 0.02, 12 + V)
    ref = oracle.logits(bits(X), bits(W))
    out = gpu_logits(X, W)
    assert_abs_close(out.cpu().double().numpy(), ref, logits_tol(X, W), "FP32 logits")
    out16 = gpu_logits(X, W, torch.bfloat16)
    assert_bf16_close(out16, ref, "BF16 logits", abs_tol=logits_tol(X, W))


def test_logits_deterministic():
    X = synth.normal_bf16((512, 2048), 1.0, 1)
    W = synth.normal_bf16((4096, 2048), 0.02, 2)
    a = gpu_logits(X, W)
    b = gpu_logits(X, W)
    assert torch.equal(a, b)


@pytest.mark.parametrize("M,K,V", [(300, 264, 1000), (17, 72, 40), (1, 8, 8), (129, 520, 2056),
                                   (1024, 128, 4096)])
def test_grad_gemms_integer_exact(M, K, V):
    dl = synth.int_bf16((M, V), 21 + M)
    X = synth.int_bf16((M, K), 22 + K)
    W = synth.int_bf16((V, K), 23 + V)
    dX = gpu_dx(dl, W).cpu().numpy()
    dW = gpu_dw(dl, X).cpu().numpy()
    refx = oracle.round_f32(oracle.dx(bits(dl), bits(W)))
    refw = oracle.round_f32(oracle.dw(bits(dl), bits(X)))
    assert np.array_equal(dX.view(np.uint32), refx.view(np.uint32)), "dX"
    assert np.array_equal(dW.view(np.uint32), refw.view(np.uint32)), "dW"


@pytest.mark.parametrize("M,K,V", [(300, 264, 1000), (17, 4096, 32776), (200, 1000, 136)])
def test_grad_gemms_random(M, K, V):
    dl = synth.normal_bf16((M, V), 1e-3, 31 + M)
    X = synth.normal_bf16((M, K), 1.0, 32 + K)
    W = synth.normal_bf16((V, K), 0.02, 33 + V)
    refx = oracle.dx(bits(dl), bits(W))
    refw = oracle.dw(bits(dl), bits(X))
    dX = gpu_dx(dl, W)
    dW = gpu_dw(dl, X)
    assert_abs_close(to_f64(dX), refx, gemm_tol(V, dl, W), "dX")
    assert_abs_close(to_f64(dW), refw, gemm_tol(M, dl, X), "dW")
    assert_bf16_close(gpu_dx(dl, W, torch.bfloat16), refx, "dX BF16", abs_tol=gemm_tol(V, dl, W))
    assert_bf16_close(gpu_dw(dl, X, torch.bfloat16), refw, "dW BF16", abs_tol=gemm_tol(M, dl, X))
    assert torch.equal(dX, gpu_dx(dl, W)) and torch.equal(dW, gpu_dw(dl, X))


@pytest.mark.parametrize("M", [128, 1024])
def test_sweep_corner_k16384_sampled(M):
    """The FP32- versus BF16-output sweep's K = 16384 shapes at full size, on
    the sweep's own inputs (X ~ N(0,1), W ~ N(0,0.02^2), 32768 vocabulary
    rows): 128 tokens take the single-token-tile CTA-pair path, 1024 tokens
    the 256 x 256 pair tiles.  Sampled token rows, FP32 and BF16 outputs."""
    c = next(c for c in synth.sweep_configs() if c.M == M and c.K == 16384)
    X = synth.normal_bf16((c.M, c.K), 1.0, c.seed)
    W = synth.normal_bf16((c.V, c.K), 0.02, c.seed + 1)
    out = gpu_logits(X, W)
    out16 = gpu_logits(X, W, torch.bfloat16)
    rows = np.array([0, 1, M // 2 + 3, M - 1])
    ref = oracle.logits(bits(X), bits(W), rows=rows)
    tr = torch.as_tensor(rows, device=DEV)
    assert_abs_close(out[tr].cpu().double().numpy(), ref, logits_tol(X, W), "FP32 logits")
    assert_bf16_close(out16[tr], ref, "BF16 logits", abs_tol=logits_tol(X, W))


def _dx_split(M, K, V):
    """How lmhead_bwd_dx splits the last (or only) wave of 256 x 256 CTA-pair
    tiles on (SMs / 2) pairs, restated: each of its rem tiles becomes a long
    part [0, B) and a short part [B, num_kb), the pairs the wave leaves idle
    taking k short parts each, B = ceil(num_kb k / (k + 1)); taken when the
    last round shortens by a tenth, and for k > 1 only after a full wave.
    Returns (rem, k, B) or None."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    tiles, pairs = (-(-K // 256)) * (-(-M // 256)), sms // 2
    nk, rem = -(-V // 64), tiles % pairs
    if nk < 2 or rem == 0:
        return None
    k = -(-rem // (pairs - rem))
    B = -(-nk * k // (k + 1))
    if (k == 1 or tiles > pairs) and k <= 8 and B < nk and 10 * max(B, k * (nk - B)) <= 9 * nk:
        return rem, k, B
    return None


def _dx_split_tiles(M, K, V):
    s = _dx_split(M, K, V)
    return s[0] if s else 0


def test_dx_last_wave_split_integer_exact():
    """2560 tokens x K = 2048: 80 pair tiles, so on 74 SM pairs the last 6 are
    each computed as two parts added into zeroed output.  Integer operands
    keep every partial sum exact, so the words must equal the oracle's;
    V = 1032 gives 17 k-blocks (parts of 9 and 8, the last one ragged)."""
    M, K, V = 2560, 2048, 1032
    if _dx_split_tiles(M, K, V) == 0:
        pytest.skip("this GPU's SM count does not split the last wave of this shape")
    dl = synth.int_bf16((M, V), 51)
    W = synth.int_bf16((V, K), 52)
    dX = gpu_dx(dl, W)
    ref = oracle.round_f32(oracle.dx(bits(dl), bits(W)))
    got = dX.cpu().numpy()
    assert np.array_equal(got, ref)  # -0.0 == +0.0: a split sum of 0 is +0
    assert torch.equal(dX, gpu_dx(dl, W))


def test_dx_last_wave_split_random_deterministic():
    M, K, V = 2560, 2048, 1032
    if _dx_split_tiles(M, K, V) == 0:
        pytest.skip("this GPU's SM count does not split the last wave of this shape")
    dl = synth.normal_bf16((M, V), 1e-3, 53)
    W = synth.normal_bf16((V, K), 0.02, 54)
    # garbage in the output beforehand: the call zeroes the rows it adds into
    out = guarded_full((M, K), float("nan"))
    st = status_word()
    lmhead.lmhead_bwd_dx(dl.to(DEV), W.to(DEV), out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rows = np.unique(np.concatenate([np.arange(0, M, 97), np.arange(M - 300, M)]))
    assert_abs_close(to_f64(out[torch.as_tensor(rows, device=DEV)]),
                     oracle.dx(bits(dl), bits(W), rows=rows), gemm_tol(V, dl, W), "dX split")
    for _ in range(3):
        assert torch.equal(out, gpu_dx(dl, W))


def test_dx_single_sparse_wave_split_integer_exact_and_deterministic():
    """Few tiles (a ragged token tile, 384 = 256 + 128, and K = 256: two pair
    tiles) on many SM pairs: both tiles are split into two parts, so four
    pairs work.  V = 65544 gives 1025 k-blocks (parts of 513 and 512, the last
    one ragged).  Integer operands keep the words exact; random operands are within
    the tolerance and bitwise repeatable."""
    M, K, V = 384, 256, 65544
    assert _dx_split_tiles(M, K, V) == 2
    dl = synth.int_bf16((M, V), 61)
    W = synth.int_bf16((V, K), 62)
    got = gpu_dx(dl, W).cpu().numpy()
    assert np.array_equal(got, oracle.round_f32(oracle.dx(bits(dl), bits(W))))
    dl = synth.normal_bf16((M, V), 1e-3, 63)
    W = synth.normal_bf16((V, K), 0.02, 64)
    out = gpu_dx(dl, W)
    rows = np.array([0, 1, 200, 255, 256, 300, M - 1])
    assert_abs_close(to_f64(out[torch.as_tensor(rows, device=DEV)]),
                     oracle.dx(bits(dl), bits(W), rows=rows), gemm_tol(V, dl, W), "dX split")
    for _ in range(2):
        assert torch.equal(out, gpu_dx(dl, W))


@pytest.mark.parametrize("M,K,V,k", [(2048, 4096, 8200, 3), (4352, 1792, 4104, 2)])
def test_dx_split_with_several_short_parts(M, K, V, k):
    """A last wave that fills most of the SM pairs after a full one: 128
    tiles (2048 tokens, K = 4096) leave 20 of 74 pairs idle in the second
    round, so each of its 54 tiles keeps a long part of 97 of its 129 k-blocks
    and the idle pairs take 3 short parts of 32 each; 119 tiles (4352 tokens,
    K = 1792) take 2 short parts per idle pair.  Integer operands: the words
    must equal the oracle's on sampled token rows (every output column, so
    every tile of those rows); random operands: within the tolerance and
    bitwise repeatable."""
    plan = _dx_split(M, K, V)
    if plan is None or plan[1] != k:
        pytest.skip("this GPU's SM count gives another split of this shape")
    rows = np.unique(np.concatenate([np.arange(0, M, 61), [M - 1]]))
    tr = torch.as_tensor(rows, device=DEV)
    dl = synth.int_bf16((M, V), 71)
    W = synth.int_bf16((V, K), 72)
    got = gpu_dx(dl, W)[tr].cpu().numpy()
    assert np.array_equal(got, oracle.round_f32(oracle.dx(bits(dl), bits(W), rows=rows)))
    dl = synth.normal_bf16((M, V), 1e-3, 73)
    W = synth.normal_bf16((V, K), 0.02, 74)
    out = gpu_dx(dl, W)
    assert_abs_close(to_f64(out[tr]), oracle.dx(bits(dl), bits(W), rows=rows),
                     gemm_tol(V, dl, W), "dX split")
    for _ in range(2):
        assert torch.equal(out, gpu_dx(dl, W))


def test_grad_gemms_large_sampled():
    """M=1024, K=4096, V=32768: sampled rows of dX and dW against the oracle."""
    M, K, V = 1024, 4096, 32768
    dl = synth.normal_bf16((M, V), 3e-5, 41)
    X = synth.normal_bf16((M, K), 1.0, 42)
    W = synth.normal_bf16((V, K), 0.02, 43)
    dX, dW = gpu_dx(dl, W), gpu_dw(dl, X)
    rng = np.random.default_rng(1239)
    rx = np.sort(rng.choice(M, 12, replace=False))
    rw = np.sort(np.concatenate([rng.choice(V, 24, replace=False), [0, V - 1]]))
    assert_abs_close(to_f64(dX[torch.as_tensor(rx, device=DEV)]),
                     oracle.dx(bits(dl), bits(W), rows=rx), gemm_tol(V, dl, W), "dX sampled")
    assert_abs_close(to_f64(dW[torch.as_tensor(rw, device=DEV)]),
                     oracle.dw(bits(dl), bits(X), vrows=rw), gemm_tol(M, dl, X), "dW sampled")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_direct_store_epilogue_on_unaligned_output(dtype):
    """An output a tensor map cannot describe (base not 16-byte aligned) takes
    the direct-store epilogue; the results are the same bits (dX here has
    three tiles, split into k-halves on both paths)."""
    M, K, V = 70, 264, 1000
    X = synth.normal_bf16((M, K), 1.0, 5)
    W = synth.normal_bf16((V, K), 0.02, 6)
    dl = synth.normal_bf16((M, V), 1e-3, 7)
    ref = gpu_logits(X, W, dtype)
    refx, refw = gpu_dx(dl, W, dtype), gpu_dw(dl, X, dtype)
    Xd, Wd, dld = X.to(DEV), W.to(DEV), dl.to(DEV)
    for shape, fn, expect in [((M, V), lambda o, s: lmhead.lmhead_fwd(Xd, Wd, o, s), ref),
                              ((M, K), lambda o, s: lmhead.lmhead_bwd_dx(dld, Wd, o, s), refx),
                              ((V, K), lambda o, s: lmhead.lmhead_bwd_dw(dld, Xd, o, s), refw)]:
        n = shape[0] * shape[1]
        buf = torch.zeros(n + 8, dtype=dtype, device=DEV)
        off = 1  # one element: 4 or 2 bytes past a 16-byte boundary
        out = buf[off:off + n].view(shape)
        assert out.data_ptr() % 16 != 0
        st = status_word()
        fn(out, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert torch.equal(out, expect)
        assert bool((buf[:off] == 0).all()) and bool((buf[off + n:] == 0).all()), "wrote outside"


@pytest.mark.parametrize("M,K,V", [(300, 264, 1000), (17, 72, 40), (1024, 128, 4096)])
def test_dw_accumulate_integer_exact(M, K, V):
    """dW += dl^T X: with integer operands and an integer starting dW the sum is
    exact, so the result equals dW0 + the exact product word for word, and
    accumulating twice adds the product twice."""
    dl = synth.int_bf16((M, V), 81 + M)
    X = synth.int_bf16((M, K), 82 + K)
    dW0 = torch.randint(-1000, 1001, (V, K), generator=torch.Generator().manual_seed(83)).float()
    prod = torch.from_numpy(oracle.dw(bits(dl), bits(X))).float()
    dW = dW0.to(DEV)
    st = status_word()
    lmhead.lmhead_bwd_dw_acc(dl.to(DEV), X.to(DEV), dW, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(dW.cpu(), dW0 + prod)
    lmhead.lmhead_bwd_dw_acc(dl.to(DEV), X.to(DEV), dW, st)
    torch.cuda.synchronize()
    assert torch.equal(dW.cpu(), dW0 + 2 * prod)


def test_dw_accumulate_random_both_epilogue_paths():
    M, K, V = 200, 1000, 136
    dl = synth.normal_bf16((M, V), 1e-3, 91)
    X = synth.normal_bf16((M, K), 1.0, 92)
    dW0 = (torch.randn((V, K), generator=torch.Generator().manual_seed(93)) * 1e-3).float()
    ref = dW0.double().numpy() + oracle.dw(bits(dl), bits(X))
    dld, Xd = dl.to(DEV), X.to(DEV)
    a = dW0.to(DEV)
    lmhead.lmhead_bwd_dw_acc(dld, Xd, a)
    # an output a tensor map cannot describe takes the per-element atomic path
    buf = torch.zeros(V * K + 1, dtype=torch.float32, device=DEV)
    b = buf[1:].view(V, K)
    b.copy_(dW0.to(DEV))
    assert b.data_ptr() % 16 != 0
    lmhead.lmhead_bwd_dw_acc(dld, Xd, b)
    torch.cuda.synchronize()
    tol = gemm_tol(M, dl, X) + 2.0 ** -23 * float(np.abs(ref).max())
    assert_abs_close(a.cpu().double().numpy(), ref, tol, "dW accumulated")
    assert torch.equal(a, b)
    assert float(buf[0]) == 0.0
