"""Parity of the cross-entropy kernels (ce_fwd, ce_bwd) with the FP64 oracle,
through the C ABI.  Stage-wise: the oracle reads the same FP32 logits the
kernels read."""
import math

import numpy as np
import pytest
import torch

import oracle
from lm_head_fp32_b200 import lmhead, synth
from helpers import assert_abs_close, assert_bf16_close, guarded_empty, loss_tol, to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_ce(x: torch.Tensor, t: torch.Tensor, g, dl_dtype=torch.float32, ignore=-100):
    """x, t on the device; g: python float (stride 0) or a [M] FP32 tensor."""
    M, V = x.shape
    st = guarded_empty((M, 4), torch.float32)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    lmhead.ce_fwd(x, t, st, ignore, status)
    gl = torch.tensor([g], dtype=torch.float32, device=DEV) if not torch.is_tensor(g) else g.to(DEV)
    dl = guarded_empty((M, V), dl_dtype)
    lmhead.ce_bwd(x, t, st, gl, dl, ignore, status)
    torch.cuda.synchronize()
    return st, dl, int(status.item())


def check_stats(st_gpu, x_cpu, t_cpu, rows=None, ignore=-100):
    ref, code = oracle.ce_fwd(x_cpu.numpy(), t_cpu.numpy(), ignore, rows=rows)
    st = st_gpu.cpu().double().numpy() if rows is None else st_gpu[torch.as_tensor(rows)].cpu().double().numpy()
    valid = code == oracle.ROW_VALID
    # m and x_y are copies of input values: exact
    assert np.array_equal(st[valid, 0], ref[valid, 0]), "row max"
    assert np.array_equal(st[valid, 2], ref[valid, 2]), "target logit"
    assert_abs_close(st[valid, 1], ref[valid, 1], 1e-5 * ref[valid, 1], "sum-exp d")
    assert_abs_close(st[:, 3], ref[:, 3], loss_tol(ref[:, 3]), "loss")
    assert (st[~valid] == 0).all(), "ignored rows must have zero stats"
    return code


def check_dl(dl_gpu, x_cpu, t_cpu, g, rows=None, ignore=-100):
    ref = oracle.ce_bwd(x_cpu.numpy(), t_cpu.numpy(), g, ignore, rows=rows)
    d = dl_gpu if rows is None else dl_gpu[torch.as_tensor(rows, device=dl_gpu.device)]
    if d.dtype == torch.float32:
        assert_abs_close(to_f64(d), ref, 1e-6, "FP32 dlogits")
    else:
        assert_bf16_close(d, ref, "BF16 dlogits")
    return ref


@pytest.mark.parametrize("M,V", [(37, 1000), (37, 1001), (5, 3), (3, 1), (64, 32776), (9, 4099)])
@pytest.mark.parametrize("dl_dtype", [torch.float32, torch.bfloat16])
def test_ce_small_shapes(M, V, dl_dtype):
    x, _ = synth.ce_logits(M, V, 4.0, 1234 + V)
    t = synth.targets(M, V, 0.1, 1234 + M)
    st, dl, status = run_ce(x.to(DEV), t.to(DEV), 1.0, dl_dtype)
    assert status == 0
    check_stats(st, x, t)
    check_dl(dl, x, t, 1.0)


def test_ce_uniform_rows_give_log_v():
    for V in (32768, 128256, 151936):
        x = torch.full((4, V), -2.5, dtype=torch.float32)
        t = torch.tensor([0, V - 1, 7, 100])
        st, dl, _ = run_ce(x.to(DEV), t.to(DEV), 1.0)
        loss = st[:, 3].cpu().double().numpy()
        assert np.all(np.abs(loss - math.log(V)) <= 1e-5 * math.log(V))
        rs = dl.double().sum(dim=1).cpu().numpy()
        assert np.all(np.abs(rs) < V * 2.0 ** -24)


def test_ce_outliers_with_targets_on_them():
    M, V = 16, 151936
    x, orows = synth.ce_logits(M, V, 4.0, 99, outlier_frac=0.5)
    t = synth.targets(M, V, 0.0, 99)
    # put some targets on a +80 and on a -80 outlier (loss ~ 0 and ~ 160)
    for r in orows.tolist()[:4]:
        pos = torch.nonzero(x[r] == 80.0).flatten()
        neg = torch.nonzero(x[r] == -80.0).flatten()
        t[r] = int(pos[0]) if (r % 2 == 0 and len(pos)) else int(neg[0]) if len(neg) else int(pos[0])
    st, dl, status = run_ce(x.to(DEV), t.to(DEV), 1.0)
    assert status == 0
    assert torch.isfinite(st).all() and torch.isfinite(dl).all()
    check_stats(st, x, t)
    check_dl(dl, x, t, 1.0)


def test_ce_bad_target_sets_status_and_zeroes_row():
    M, V = 6, 500
    x, _ = synth.ce_logits(M, V, 2.0, 5)
    t = torch.tensor([3, 500, -100, -1, 499, 10**12])
    st, dl, status = run_ce(x.to(DEV), t.to(DEV), 1.0)
    assert status & lmhead.DEV_BAD_TARGET
    for r in (1, 2, 3, 5):
        assert (st[r] == 0).all() and (dl[r] == 0).all()
    check_stats(st, x, t)
    check_dl(dl, x, t, 1.0)


def test_ce_ignored_rows_are_not_read():
    """Ignored rows hold NaN here: the kernels never read them (zero statistics
    and gradient, no status bit), and the other rows are unaffected.  A batch
    in which every row is ignored gives zeros throughout."""
    M, V = 70, 3000
    x, _ = synth.ce_logits(M, V, 4.0, 21)
    t = synth.targets(M, V, 0.0, 21)
    t[1::2] = -100
    x[1::2] = float("nan")
    st, dl, status = run_ce(x.to(DEV), t.to(DEV), 1.0, torch.bfloat16)
    assert status == 0
    assert (st[1::2] == 0).all() and (dl[1::2].float() == 0).all()
    check_stats(st, x, t)
    check_dl(dl, x, t, 1.0)
    t[:] = -100
    st, dl, status = run_ce(x.to(DEV), t.to(DEV), 1.0)
    assert status == 0
    assert (st == 0).all() and (dl == 0).all()


def test_ce_custom_ignore_index_and_per_row_grad():
    M, V = 33, 2048
    x, _ = synth.ce_logits(M, V, 3.0, 8)
    t = synth.targets(M, V, 0.0, 8)
    t[::5] = 7                               # ignore_index = 7 here
    g = torch.rand(M, generator=torch.Generator().manual_seed(3)).to(torch.float32)
    st, dl, status = run_ce(x.to(DEV), t.to(DEV), g, ignore=7)
    assert status == 0
    check_stats(st, x, t, ignore=7)
    ref = oracle.ce_bwd(x.numpy(), t.numpy(), g.numpy(), 7)
    assert_abs_close(to_f64(dl), ref, 1e-6, "per-row grad dlogits")


def test_ce_bwd_in_place_matches_out_of_place():
    M, V = 40, 5000
    x, _ = synth.ce_logits(M, V, 4.0, 17)
    t = synth.targets(M, V, 0.05, 17)
    xd, td = x.to(DEV), t.to(DEV)
    st, dl, _ = run_ce(xd, td, 0.5)
    buf = xd.clone()
    gl = torch.tensor([0.5], device=DEV)
    lmhead.ce_bwd(buf, td, st, gl, buf)     # dlogits written over the logits
    torch.cuda.synchronize()
    assert torch.equal(buf, dl)


def test_ce_deterministic():
    x, _ = synth.ce_logits(64, 32768, 4.0, 3)
    t = synth.targets(64, 32768, 0.0, 3)
    a = run_ce(x.to(DEV), t.to(DEV), 1.0)
    b = run_ce(x.to(DEV), t.to(DEV), 1.0)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_ce_wide_outlier_config_sampled():
    """8192 x 151936 FP32 rows, N(0,4^2), 1% outlier rows (16 entries of +-80),
    1% ignored rows; FP32 then BF16 dlogits.  Sampled rows against the oracle,
    every output checked finite."""
    cfg = synth.CE_WIDE
    x, t, orows = cfg.make(device=DEV)
    td = t.to(DEV)
    st, dl32, status = run_ce(x, td, 1.0, torch.float32)
    assert status == 0
    assert bool(torch.isfinite(st).all()) and bool(torch.isfinite(dl32).all())
    ign = torch.nonzero(t == -100).flatten()
    rng = np.random.default_rng(cfg.seed + 5)
    rows = np.unique(np.concatenate([rng.choice(cfg.rows, 24, replace=False), orows.numpy()[:24],
                                     ign.numpy()[:8]]))
    xs = x[torch.as_tensor(rows, device=DEV)].cpu()
    ts = t[torch.as_tensor(rows)]
    check_stats(st[torch.as_tensor(rows, device=DEV)], xs, ts)
    ref = oracle.ce_bwd(xs.numpy(), ts.numpy(), 1.0)
    assert_abs_close(to_f64(dl32[torch.as_tensor(rows, device=DEV)]), ref, 1e-6, "FP32 dlogits (wide)")
    valid = (t != -100).to(DEV)
    rsum = dl32.sum(dim=1)
    assert float(rsum[valid].abs().max()) < cfg.cols * 2.0 ** -24
    del dl32
    _, dl16, status = run_ce(x, td, 1.0, torch.bfloat16)
    assert status == 0 and bool(torch.isfinite(dl16).all())
    assert_bf16_close(dl16[torch.as_tensor(rows, device=DEV)], ref, "BF16 dlogits (wide)")
