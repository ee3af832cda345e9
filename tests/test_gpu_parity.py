"""GPU parity: the CUDA path (through the C ABI) against the FP64 oracle on the
same seeded BF16 inputs.

Gates (relative RMSE = ||x - x_ref|| / ||x_ref|| over the compared elements,
FP64): output and dV <= 1e-2; dQ, dK and dBias <= 2e-2.  Small cases compare
every element; crop-sized cases compare sampled pair rows (every element of
those rows) and sampled dBias rows (each a sum over all N pair rows), at the
same launch configuration the benchmark times.
Repeatability: fixed inputs run 5 times give bitwise-identical outputs and
gradients ("TurboPairFormer: более быстрое, стабильное и точное дообучение
OpenFold3", section "Воспроизводимость и стабильность").
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from triangle_attention_biomolecular_b200 import _binding as Bd
from triangle_attention_biomolecular_b200 import api
from triangle_attention_biomolecular_b200 import synthetic as S

pytestmark = pytest.mark.gpu

GATES = {"out": 1e-2, "dv": 1e-2, "dq": 2e-2, "dk": 2e-2, "dbias": 2e-2}


def rel(a, b):
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _nan_like(t):
    return torch.full_like(t, float("nan"))


def run_gpu(x, orientation, flags=0, bias_row_pad=None, mask=None, keep=False):
    """Forward then backward through the C ABI.  Every output buffer (o, resid,
    lse, dq, dk, dv, dbias) is filled with NaN before the call and the workspace
    with 0xFF bytes (NaN as FP32), so a result the kernels did not write, or a
    workspace word read before it is written, cannot pass as a value.
    ``mask``: overrides x["mask"] (e.g. a stride-0 broadcast view)."""
    dev = torch.device("cuda")
    q, k, v, do = (S.to_attention_frame(x[n].to(dev), orientation) for n in ("q", "k", "v", "dout"))
    bias = x["bias"].to(dev)
    if bias_row_pad is None and bias.shape[-1] % 8:
        bias_row_pad = (bias.shape[-1] + 7) // 8 * 8  # the ABI wants row strides of 8-element multiples
    if bias_row_pad is not None:  # same values, rows padded on the device (row stride bias_row_pad)
        N = bias.shape[-1]
        buf = torch.zeros(bias.shape[:-1] + (bias_row_pad,), dtype=bias.dtype, device=dev)
        buf[..., :N] = bias
        bias = buf[..., :N]
    if mask is None and x["mask"] is not None:
        mask = x["mask"].to(dev)
    Bn, N, _, H, d = q.shape
    o, r = _nan_like(q), _nan_like(q)
    lse = torch.full((Bn, H, N, N), float("nan"), dtype=torch.float32, device=dev)
    Bd.tri_attn_fwd(q, k, v, bias, mask, o, r, lse)
    dq, dk, dv = _nan_like(q), _nan_like(k), _nan_like(v)
    Npad = (N + 7) // 8 * 8  # dbias rows padded to a 16-byte multiple
    db = torch.full((Bn, H, N, Npad), float("nan"), dtype=torch.bfloat16, device=dev)[..., :N]
    ws = torch.full((Bd.tri_attn_bwd_workspace_bytes(Bn, N, H, d),), 0xFF, dtype=torch.uint8, device=dev)
    Bd.tri_attn_bwd(q, k, v, bias, mask, o, r, lse, do, dq, dk, dv, db, ws, 0.0, flags)
    torch.cuda.synchronize()
    st, word = Bd.tri_attn_device_error(True)
    assert st == Bd.TRI_ATTN_OK, f"device error word {word:#x}"
    cpu = lambda t: t.float().cpu()
    res = {"out": cpu(o), "resid": cpu(r), "lse": lse.cpu(), "dq": cpu(dq), "dk": cpu(dk), "dv": cpu(dv),
           "dbias": cpu(db)}
    if keep:  # the device buffers stay alive with the result (no later run can reuse them)
        res["_device"] = (o, r, lse, dq, dk, dv, db, ws)
    return res


def oracle_inputs(x, orientation):
    f = lambda n: S.to_attention_frame(x[n], orientation)
    return f("q"), f("k"), f("v"), x["bias"], x["mask"], f("dout")


def check_full(x, got, orientation="start"):
    q, k, v, bias, mask, do = oracle_inputs(x, orientation)
    out, lse = O.fwd(q, k, v, bias, mask)
    dq, dk, dv, db = O.bwd(q, k, v, bias, mask, do)
    ref = {"out": out, "dq": dq, "dk": dk, "dv": dv, "dbias": db}
    errs = {n: rel(got[n].numpy(), ref[n]) for n in ref}
    for n, e in errs.items():
        assert np.all(np.isfinite(got[n].numpy())), n
        assert e <= GATES[n], f"{n}: rel-RMSE {e:.3e} > {GATES[n]}"
    assert np.max(np.abs(got["lse"].numpy() - lse)) < 2e-3
    return errs, ref


def check_sampled(x, got, rows, sel, orientation="start"):
    q, k, v, bias, mask, do = oracle_inputs(x, orientation)
    out, lse = O.fwd(q, k, v, bias, mask, rows=rows)
    dq, dk, dv = O.bwd_rows(q, k, v, bias, mask, do, rows=rows)
    db = O.dbias(q, k, v, bias, mask, do, sel=sel)
    errs = {}
    for n, ref in (("out", out), ("dq", dq), ("dk", dk), ("dv", dv)):
        g = np.stack([got[n].numpy()[b, i] for b, i in rows])
        r = np.stack([ref[b, i] for b, i in rows])
        assert np.all(np.isfinite(g)), n
        errs[n] = rel(g, r)
    g = np.stack([got["dbias"].numpy()[b, h, j] for b, h, j in sel])
    r = np.stack([db[b, h, j] for b, h, j in sel])
    errs["dbias"] = rel(g, r)
    for n, e in errs.items():
        assert e <= GATES[n], f"{n}: rel-RMSE {e:.3e} > {GATES[n]}"
    lg = np.stack([got["lse"].numpy()[b, :, i] for b, i in rows])
    lr = np.stack([lse[b, :, i] for b, i in rows])
    assert np.max(np.abs(lg - lr)) < 2e-3
    return errs


def sample_rows(wl, n, seed):
    rng = np.random.default_rng(seed)
    rows = {(0, 0), (wl.B - 1, wl.N - 1)}
    while len(rows) < n:
        rows.add((int(rng.integers(wl.B)), int(rng.integers(wl.N))))
    sel = {(0, 0, 0), (wl.B - 1, wl.H - 1, wl.N - 1)}
    while len(sel) < n:
        sel.add((int(rng.integers(wl.B)), int(rng.integers(wl.H)), int(rng.integers(wl.N))))
    return sorted(rows), sorted(sel)


# ---------------------------------------------------------------------------
# full comparisons on small cases (several tiles, ragged tails)
# ---------------------------------------------------------------------------

def test_tiny_full():
    x = S.make_inputs(S.TINY, S.seed_for(0, 0))
    got = run_gpu(x, "start")
    errs, ref = check_full(x, got)
    # resid is the BF16 rounding residual of the FP32 result: at most half a BF16
    # ulp of o, and o + resid is closer to the exact result than o alone
    o, r = got["out"].numpy(), got["resid"].numpy()
    half_ulp = np.abs(o) * 2.0 ** -8 + 1e-30
    assert np.all(np.abs(r) <= half_ulp * 1.0001)
    assert rel(o + r, ref["out"]) < 0.75 * errs["out"]


@pytest.mark.parametrize("d", [32, 64])
def test_two_tiles_ragged_mask_full(d):
    wl = S.Workload("small ragged", 2, 136, 2, d, mask="ragged", len_lo=70, len_hi=136)
    x = S.make_inputs(wl, 77 + d)
    check_full(x, run_gpu(x, "start"))


def test_odd_N_with_padded_bias_rows():
    # N odd (the last pair of rows has a single row) and not a multiple of 8: the
    # bias lives in a [.., N, 40] buffer so its row stride stays 16-byte aligned
    wl = S.Workload("odd", 1, 37, 2, 32, mask="ragged", len_lo=20, len_hi=37)
    x = S.make_inputs(wl, 5)
    check_full(x, run_gpu(x, "start", bias_row_pad=40))


def test_ending_node_full():
    wl = S.Workload("end small", 1, 72, 2, 32, mask="ragged", len_lo=40, len_hi=72, orientation="end")
    x = S.make_inputs(wl, 9)
    check_full(x, run_gpu(x, "end"), "end")


def test_no_mask_equals_zero_mask_bitwise():
    wl = S.Workload("zeros", 1, 96, 2, 32, mask="zeros")
    x = S.make_inputs(wl, 3)
    a = run_gpu(x, "start")
    x2 = dict(x)
    x2["mask"] = None
    b = run_gpu(x2, "start")
    for n in a:
        assert torch.equal(a[n], b[n]), n


# ---------------------------------------------------------------------------
# crop-sized workloads: sampled rows at full size
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("wl,idx", [(S.CROP384, 1), (S.CROP640, 2),
                                    (S.CROP640.with_(orientation="end"), 2)])
def test_crop_sampled(wl, idx):
    x = S.make_inputs(wl, S.seed_for(idx, 0))
    got = run_gpu(x, wl.orientation)
    rows, sel = sample_rows(wl, 6, idx)
    check_sampled(x, got, rows, sel, wl.orientation)


def _bits(t):
    return t.view(torch.int32)


def test_crop768_sampled_and_bitwise_repeatable():
    """Five runs of the headline workload, each into fresh NaN-filled buffers that
    all stay allocated until the comparison (so no run can inherit another's
    bits): every output and gradient is bitwise identical across the five."""
    wl = S.CROP768
    x = S.make_inputs(wl, S.seed_for(3, 0))
    runs = [run_gpu(x, "start", keep=True) for _ in range(5)]
    ptrs = {t.data_ptr() for r in runs for t in r["_device"]}
    assert len(ptrs) == 5 * 8, "the five runs must not share device buffers"
    for r in runs[1:]:  # FP32 copies of the BF16 results keep every bit, the sign of zero included
        for n in ("out", "resid", "lse", "dq", "dk", "dv", "dbias"):
            assert torch.equal(_bits(r[n]), _bits(runs[0][n])), n
    for n in ("out", "dq", "dk", "dv", "dbias"):
        assert torch.isfinite(runs[0][n]).all(), n
    rows, sel = sample_rows(wl, 6, 3)
    check_sampled(x, runs[0], rows, sel)


@pytest.mark.parametrize("N", S.SWEEP_NS)
@pytest.mark.parametrize("d", S.SWEEP_DS)
def test_sweep_sampled(N, d):
    wl = S.sweep(N, d)
    x = S.make_inputs(wl, S.seed_for(4, 10 * d + N // 128))
    got = run_gpu(x, "start")
    rows, sel = sample_rows(wl, 4, N + d)
    check_sampled(x, got, rows, sel)


# ---------------------------------------------------------------------------
# residual compensation variant and the bounded-wait path
# ---------------------------------------------------------------------------

def test_uncompensated_variant_runs_and_stays_within_gates():
    wl = S.Workload("ablation", 1, 128, 4, 32)
    x = S.make_inputs(wl, 11)
    got = run_gpu(x, "start", flags=Bd.TRI_ATTN_BWD_NO_RESIDUAL)
    check_full(x, got)


@pytest.mark.parametrize("wl", [S.Workload("ablation N=256 bias 2N(0,1)", 1, 256, 4, 32, bias_std=2.0, mask="zeros"),
                                S.Workload("ablation N=200 ragged", 1, 200, 4, 32, mask="ragged", len_lo=150,
                                           len_hi=200)],
                         ids=["N256", "N200ragged"])
def test_residual_compensation_ablation(wl, capsys):
    """The output-rounding residual (D formed in FP32 from o + resid, versus from the
    BF16 output o alone; TurboPairFormer pages, "residual compensation").  Measured
    against the FP64 oracle: dV does not involve D and must be bitwise identical;
    dQ, dK and dBias must come out closer to the exact gradients with the residual."""
    x = S.make_inputs(wl, 21)
    comp = run_gpu(x, "start")
    unc = run_gpu(x, "start", flags=Bd.TRI_ATTN_BWD_NO_RESIDUAL)
    assert torch.equal(comp["dv"], unc["dv"])
    q, k, v, bias, mask, do = oracle_inputs(x, "start")
    dq, dk, dv, db = O.bwd(q, k, v, bias, mask, do)
    ref = {"dq": dq, "dk": dk, "dbias": db}
    e_c = {n: rel(comp[n].numpy(), ref[n]) for n in ref}
    e_u = {n: rel(unc[n].numpy(), ref[n]) for n in ref}
    with capsys.disabled():
        print(f"\n[{wl.name}] rel-RMSE vs FP64, compensated / uncompensated: " +
              ", ".join(f"{n} {e_c[n]:.3e} / {e_u[n]:.3e} ({100 * (1 - e_c[n] / e_u[n]):+.1f}%)" for n in ref))
    for n in ref:
        assert e_c[n] <= GATES[n] and e_u[n] <= GATES[n], n
        assert e_c[n] < e_u[n], f"{n}: residual did not reduce the error ({e_c[n]:.3e} vs {e_u[n]:.3e})"


def test_bounded_wait_expires_and_context_survives():
    Bd.tri_attn_device_error(True)
    Bd.tri_attn_set_wait_limit_ns(2_000_000)  # 2 ms
    try:
        Bd.tri_attn_selftest_expire_wait()
        torch.cuda.synchronize()
        st, word = Bd.tri_attn_device_error(True)
        assert st == Bd.TRI_ATTN_ERR_DEVICE_TIMEOUT and word != 0
    finally:
        Bd.tri_attn_set_wait_limit_ns(2_000_000_000)
    # the context is still usable
    x = S.make_inputs(S.TINY, 1)
    check_full(x, run_gpu(x, "start"))


# ---------------------------------------------------------------------------
# the method's edge cases: masked keys, one and two keys, the largest N,
# broadcast masks, the autograd entry point and a backward from saved state
# ---------------------------------------------------------------------------

def _assert_masked_keys_exactly_zero(x, got, masked):
    """masked: bool [B, N] over keys.  A masked key has probability exactly 0 in
    FP32 (exp of about -1e9), so it receives exactly zero dK, dV and dBias (the
    survey's 'masking in bwd' pin, asserted here on the GPU results)."""
    for b in range(masked.shape[0]):
        ks = torch.nonzero(masked[b]).flatten()
        if ks.numel() == 0:
            continue
        for n in ("dk", "dv"):
            sub = got[n][b][:, ks]
            assert torch.equal(sub, torch.zeros_like(sub)), f"{n}: batch {b} masked keys not exactly zero"
        sub = got["dbias"][b][..., ks]
        assert torch.equal(sub, torch.zeros_like(sub)), f"dbias: batch {b} masked keys not exactly zero"
    for n in ("out", "dq", "dk", "dv", "dbias"):
        assert torch.isfinite(got[n]).all(), n


@pytest.mark.parametrize("wl,seed", [
    (S.Workload("ragged N=200 L=150", 1, 200, 4, 32, mask="ragged", len_lo=150, len_hi=150), 31),
    (S.Workload("ragged B=2 N=300", 2, 300, 2, 32, mask="ragged", len_lo=140, len_hi=290), 32),
    (S.Workload("ragged d=64 N=200", 1, 200, 2, 64, mask="ragged", len_lo=100, len_hi=180), 33),
], ids=["N200L150", "B2N300", "d64N200"])
def test_masked_keys_get_exactly_zero_gradients(wl, seed):
    x = S.make_inputs(wl, seed)
    got = run_gpu(x, "start")
    L = x["lengths"]
    masked = torch.arange(wl.N).view(1, -1) >= L.view(-1, 1)
    _assert_masked_keys_exactly_zero(x, got, masked)
    check_full(x, got)


def test_mask_confined_to_one_key_tile():
    """A mask that is -1e9 for keys 200..229 only (inside the second 128-key tile):
    the first and third tiles take the mask-free path (where a quarter of the
    exponentials run on the FMA pipe), the second the masked path; the masked
    keys still get exactly zero gradients."""
    wl = S.Workload("one masked tile", 1, 384, 2, 32, mask="zeros")
    x = S.make_inputs(wl, 34)
    m = torch.zeros(1, 384, 384)
    m[..., 200:230] = S.MASK_NEG
    x["mask"] = m
    got = run_gpu(x, "start")
    masked = torch.zeros(1, 384, dtype=torch.bool)
    masked[0, 200:230] = True
    _assert_masked_keys_exactly_zero(x, got, masked)
    check_full(x, got)


def test_crop384_masked_keys_exactly_zero():
    x = S.make_inputs(S.CROP384, S.seed_for(1, 1))
    got = run_gpu(x, "start")
    masked = torch.arange(S.CROP384.N).view(1, -1) >= x["lengths"].view(-1, 1)
    assert masked.any()
    _assert_masked_keys_exactly_zero(x, got, masked)


def test_single_key():
    """N = 1: the softmax over one key is 1, so out = v and dV = dout bit for bit
    (P is 1 to within a few FP32 ulps, exactly 1 once rounded to BF16), resid is
    at most that FP32 error, lse = the one score, and dQ, dK, dBias vanish
    (dS = P (dP - D) with dP = D up to FP32 summation order)."""
    for d in (32, 64):
        wl = S.Workload("N=1", 2, 1, 3, d)
        x = S.make_inputs(wl, 35 + d)
        got = run_gpu(x, "start", bias_row_pad=8)
        assert torch.equal(got["out"], x["v"].float())
        # resid is a BF16 rounding residual: at most half a BF16 ulp of o
        assert torch.all(got["resid"].abs() <= 2.0 ** -8 * got["out"].abs() * 1.0001 + 1e-30)
        assert torch.equal(got["dv"], x["dout"].float())
        q, k, v, bias, mask, do = oracle_inputs(x, "start")
        _, lse = O.fwd(q, k, v, bias, mask)
        assert np.max(np.abs(got["lse"].numpy() - lse)) < 2e-3
        for n in ("dq", "dk", "dbias"):
            assert torch.isfinite(got[n]).all() and got[n].abs().max().item() < 1e-3, n


def test_two_keys_full():
    # both keys valid (with one of two masked the row is the single-key case above,
    # whose exact dQ, dK, dBias are zero and have no relative error to speak of)
    wl = S.Workload("N=2", 2, 2, 3, 32, mask="zeros")
    x = S.make_inputs(wl, 37)
    check_full(x, run_gpu(x, "start", bias_row_pad=8))


def test_broadcast_mask_stride_zero():
    """A [B,1,N] key mask expanded over rows i (stride 0 on the row axis), as the
    header allows: equal bit for bit to the same mask materialised, and to the
    oracle within the gates."""
    wl = S.Workload("broadcast mask", 2, 136, 2, 32, mask="ragged", len_lo=70, len_hi=120)
    x = S.make_inputs(wl, 38)
    dev = torch.device("cuda")
    row = x["mask"][:, :1, :].to(dev)          # [B,1,N]
    bmask = row.expand(wl.B, wl.N, wl.N)       # stride (N, 0, 1)
    assert bmask.stride(1) == 0
    a = run_gpu(x, "start", mask=bmask)
    b = run_gpu(x, "start")
    for n in a:
        assert torch.equal(a[n], b[n]), n
    check_full(x, a)


def test_largest_n_sampled_rows():
    """N = 4096, the largest size the library accepts (32 key tiles; dQ goes
    through the per-CTA FP32 slots).  Inputs are drawn on the device; the oracle
    runs on single pair rows (out, dq, dk, dv of two rows) and streams all 4096
    rows for two dBias rows."""
    wl = S.Workload("N=4096", 1, 4096, 1, 32, mask="ragged", len_lo=3000, len_hi=4096)
    dev = torch.device("cuda")
    x = S.make_inputs_device(wl, 39, dev)
    q, k, v, do, bias, mask = x["q"], x["k"], x["v"], x["dout"], x["bias"], x["mask"]
    N, H, d = wl.N, wl.H, wl.d
    o, r = _nan_like(q), _nan_like(q)
    lse = torch.full((1, H, N, N), float("nan"), dtype=torch.float32, device=dev)
    Bd.tri_attn_fwd(q, k, v, bias, mask, o, r, lse)
    dq, dk, dv = _nan_like(q), _nan_like(q), _nan_like(q)
    db = torch.full((1, H, N, N), float("nan"), dtype=torch.bfloat16, device=dev)
    ws = torch.full((Bd.tri_attn_bwd_workspace_bytes(1, N, H, d),), 0xFF, dtype=torch.uint8, device=dev)
    Bd.tri_attn_bwd(q, k, v, bias, mask, o, r, lse, do, dq, dk, dv, db, ws)
    torch.cuda.synchronize()
    st, word = Bd.tri_attn_device_error(True)
    assert st == Bd.TRI_ATTN_OK, f"device error word {word:#x}"
    for t, n in ((o, "out"), (dq, "dq"), (dk, "dk"), (dv, "dv"), (db, "dbias")):
        assert torch.isfinite(t).all().item(), n
    bias_c = bias[0].cpu()
    rows = [0, 2873]
    for i in rows:
        m = mask[0, i].cpu()
        ref = O.row(q[0, i].cpu(), k[0, i].cpu(), v[0, i].cpu(), bias_c, m, do[0, i].cpu())
        got = [o[0, i], lse[0, :, i], dq[0, i], dk[0, i], dv[0, i]]
        for n, g, rr in zip(("out", "lse", "dq", "dk", "dv"), got, ref):
            g = g.float().cpu().numpy()
            if n == "lse":
                assert np.max(np.abs(g - rr)) < 2e-3
            else:
                assert rel(g, rr) <= GATES[n], f"row {i} {n}: rel-RMSE {rel(g, rr):.3e}"
    qc, kc, vc, doc, mc = (t[0].cpu() for t in (q, k, v, do, mask))
    get = lambda i: (qc[i], kc[i], vc[i], mc[i], doc[i])
    for h, j in [(0, 0), (0, 3001)]:
        ref = O.dbias_streamed(get, bias_c, h, j)
        g = db[0, h, j].float().cpu().numpy()
        assert rel(g, ref) <= GATES["dbias"], f"dbias row {j}: rel-RMSE {rel(g, ref):.3e}"


@pytest.mark.parametrize("orientation", ["start", "end"])
def test_autograd_entry_point(orientation):
    """The user-facing ``triangle_attention`` through ``torch.autograd.backward``
    (the call a model makes), both orientations, against the oracle."""
    wl = S.Workload("autograd", 1, 136, 2, 32, mask="ragged", len_lo=90, len_hi=136, orientation=orientation)
    x = S.make_inputs(wl, 40)
    dev = torch.device("cuda")
    q, k, v, bias = (x[n].to(dev).requires_grad_(True) for n in ("q", "k", "v", "bias"))
    mask = x["mask"].to(dev)
    out = api.triangle_attention(q, k, v, bias, mask, orientation=orientation)
    assert out.shape == q.shape and out.dtype == torch.bfloat16
    loss = (out.float() * x["dout"].to(dev).float()).sum()
    torch.autograd.backward(loss)
    torch.cuda.synchronize()
    qo, ko, vo, bo, mo, doo = (x[n] for n in ("q", "k", "v", "bias", "mask", "dout"))
    if orientation == "start":
        ref_out, _ = O.fwd(qo, ko, vo, bo, mo)
        ref = O.bwd(qo, ko, vo, bo, mo, doo)
    else:
        ref_out, _ = O.ending_fwd(qo, ko, vo, bo, mo)
        ref = O.ending_bwd(qo, ko, vo, bo, mo, doo)
    assert rel(out.detach().float().cpu().numpy(), ref_out) <= GATES["out"]
    for n, g, rr in zip(("dq", "dk", "dv", "dbias"), (q.grad, k.grad, v.grad, bias.grad), ref):
        e = rel(g.float().cpu().numpy(), rr)
        assert e <= GATES[n], f"{n}: rel-RMSE {e:.3e}"
    # a plain out.sum() hands the backward an expanded (stride-0) gradient
    q.grad = None
    out2 = api.triangle_attention(q, k, v, bias, mask, orientation=orientation)
    out2.float().sum().backward()
    assert torch.isfinite(q.grad.float()).all()


def test_backward_from_saved_state_is_bitwise_equal():
    """The saved state (o, resid, lse) is everything the backward needs: a backward
    from a copy kept on the host across unrelated launches equals a backward right
    after a fresh forward, bit for bit (checkpoint-and-resume of the step)."""
    wl = S.Workload("saved state", 1, 256, 4, 32, mask="ragged", len_lo=180, len_hi=256)
    x = S.make_inputs(wl, 41)
    dev = torch.device("cuda")
    q, k, v, do, bias = (x[n].to(dev) for n in ("q", "k", "v", "dout", "bias"))
    mask = x["mask"].to(dev)
    o, r, lse = api.forward(q, k, v, bias, mask)
    saved = tuple(t.cpu() for t in (o, r, lse))
    del o, r, lse
    y = S.make_inputs(wl, 42)  # unrelated work in between
    run_gpu(y, "start")
    o2, r2, lse2 = (t.to(dev) for t in saved)
    from_saved = api.backward(q, k, v, bias, mask, o2, r2, lse2, do)
    o3, r3, lse3 = api.forward(q, k, v, bias, mask)
    fresh = api.backward(q, k, v, bias, mask, o3, r3, lse3, do)
    torch.cuda.synchronize()
    for a, b in zip((o2, r2, lse2), (o3, r3, lse3)):
        assert torch.equal(a, b)
    for n, a, b in zip(("dq", "dk", "dv", "dbias"), from_saved, fresh):
        assert torch.equal(a, b), n
