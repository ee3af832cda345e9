"""Pins for the FP64 oracle, against things other than the oracle itself.

* A library routine: with the pair bias and the key mask folded into one
  additive attention mask, every (b, i, h) problem is textbook scaled
  dot-product attention -> ``torch.nn.functional.scaled_dot_product_attention``
  in FP64 on CPU, and torch autograd through it for all four gradients.
* Closed forms and invariants of softmax attention (one-hot values read the
  probabilities back; constant values pass through; per-row shifts of the
  bias or mask change nothing; probability rows sum to one; masked keys get
  exactly zero probability and gradient; every dbias row sums to zero).
* FP64 central finite differences of L = sum(dout * out) for dq, dk, dv, dbias.
* Brute force: the definition as scalar Python loops on tiny sizes.
* Planted mistakes: each deliberate error the C oracle can be switched into is
  caught by at least one of these pins.

The gradient pins follow the pages' accuracy protocol -- an FP64 reference on
the identical inputs ("TurboPairFormer: более быстрое, стабильное и точное
дообучение OpenFold3", section "Точность").
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import oracle as O


def _rand(seed, B, N, H, d, mask_kind="none", bias_std=1.0):
    g = torch.Generator().manual_seed(seed)
    shp = (B, N, N, H, d)
    q = torch.randn(shp, generator=g, dtype=torch.float64)
    k = torch.randn(shp, generator=g, dtype=torch.float64)
    v = torch.randn(shp, generator=g, dtype=torch.float64)
    do = torch.randn(shp, generator=g, dtype=torch.float64)
    bias = torch.randn((B, H, N, N), generator=g, dtype=torch.float64) * bias_std
    mask = None
    if mask_kind == "ragged":
        L = torch.randint(max(1, N // 2), N + 1, (B,), generator=g)
        kidx = torch.arange(N).view(1, 1, N)
        mask = torch.where(kidx >= L.view(-1, 1, 1), -1e9, 0.0).expand(B, N, N).contiguous()
    elif mask_kind == "random":
        mask = torch.randn((B, N, N), generator=g, dtype=torch.float64)
    return q, k, v, do, bias, mask


def _sdpa(q, k, v, bias, mask, scale, need_grad=False):
    """Library path: SDPA over the (b, i, h) batch with attn_mask = bias + mask."""
    B, N, _, H, d = q.shape
    qq, kk, vv = (x.permute(0, 1, 3, 2, 4).reshape(B * N, H, N, d) for x in (q, k, v))
    am = bias.unsqueeze(1).expand(B, N, H, N, N)
    if mask is not None:
        am = am + mask.view(B, N, 1, 1, N)
    am = am.reshape(B * N, H, N, N)
    out = F.scaled_dot_product_attention(qq, kk, vv, attn_mask=am, scale=scale)
    return out.reshape(B, N, H, N, d).permute(0, 1, 3, 2, 4)


def _sdpa_lse(q, k, bias, mask, scale):
    s = torch.einsum("bijhc,bikhc->bhijk", q, k) * scale + bias.unsqueeze(2)
    if mask is not None:
        s = s + mask.view(mask.shape[0], 1, mask.shape[1], 1, mask.shape[2])
    return torch.logsumexp(s, dim=-1)  # [B,H,N(i),N(j)]


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300)


CASES = [(1, 5, 2, 4, "none"), (2, 8, 2, 4, "ragged"), (1, 16, 3, 8, "random"), (1, 32, 4, 32, "none")]


@pytest.mark.parametrize("B,N,H,d,mk", CASES)
def test_fwd_matches_library_sdpa(B, N, H, d, mk):
    q, k, v, do, bias, mask = _rand(11, B, N, H, d, mk)
    scale = 1.0 / np.sqrt(d)
    out, lse = O.fwd(q, k, v, bias, mask, scale)
    ref = _sdpa(q, k, v, bias, mask, scale).numpy()
    assert _rel(out, ref) < 1e-12
    assert _rel(lse, _sdpa_lse(q, k, bias, mask, scale).numpy()) < 1e-13


@pytest.mark.parametrize("B,N,H,d,mk", CASES[:3])
def test_bwd_matches_torch_autograd(B, N, H, d, mk):
    q, k, v, do, bias, mask = _rand(12, B, N, H, d, mk)
    scale = 1.0 / np.sqrt(d)
    qt, kt, vt, bt = (x.clone().requires_grad_(True) for x in (q, k, v, bias))
    out = _sdpa(qt, kt, vt, bt, mask, scale)
    (out * do).sum().backward()
    dq, dk, dv, db = O.bwd(q, k, v, bias, mask, do, scale)
    assert _rel(dq, qt.grad.numpy()) < 1e-11
    assert _rel(dk, kt.grad.numpy()) < 1e-11
    assert _rel(dv, vt.grad.numpy()) < 1e-11
    assert _rel(db, bt.grad.numpy()) < 1e-11


def test_one_hot_values_read_back_probabilities():
    # d == N and v[b,i,k,h,:] = e_k  =>  out[b,i,j,h,:] = p[b,i,h,j,:]
    B, N, H = 1, 6, 2
    q, k, _, _, bias, mask = _rand(13, B, N, H, N, "ragged")
    v = torch.zeros(B, N, N, H, N, dtype=torch.float64)
    for kk in range(N):
        v[:, :, kk, :, kk] = 1.0
    out, lse = O.fwd(q, k, v, bias, mask)
    p = out  # [B,N(i),N(j),H,N(k)]
    assert np.all(p >= 0)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-14)
    masked = (mask.numpy() < -1e8)  # [B,N(i),N(k)]
    for b in range(B):
        for i in range(N):
            assert np.all(p[b, i][:, :, masked[b, i]] == 0.0)
    # q = 0: p = softmax(bias[j,:] + mask[i,:]), from scipy's softmax
    from scipy.special import softmax
    out0, _ = O.fwd(torch.zeros_like(q), k, v, bias, mask)
    for b in range(B):
        for i in range(N):
            for h in range(H):
                ref = softmax(bias[b, h].numpy() + mask[b, i].numpy()[None, :], axis=-1)
                np.testing.assert_allclose(out0[b, i, :, h, :], ref, rtol=0, atol=1e-15)


def test_closed_forms_and_shift_invariance():
    B, N, H, d = 1, 7, 2, 5
    q, k, v, _, bias, mask = _rand(14, B, N, H, d, "random")
    # constant values pass through unchanged
    vc = torch.full_like(v, 0.375)
    out, _ = O.fwd(q, k, vc, bias, mask)
    np.testing.assert_allclose(out, 0.375, rtol=0, atol=1e-15)
    # shifting bias row j by c_j, or mask row i by c_i, leaves out unchanged; lse shifts
    out0, lse0 = O.fwd(q, k, v, bias, mask)
    cj = torch.randn(B, H, N, 1, dtype=torch.float64)
    out1, lse1 = O.fwd(q, k, v, bias + cj, mask)
    assert _rel(out1, out0) < 1e-13
    np.testing.assert_allclose(lse1 - lse0, np.broadcast_to(cj.numpy()[:, :, None, :, 0], lse0.shape),
                               atol=1e-12)
    ci = torch.randn(B, N, 1, dtype=torch.float64)
    out2, _ = O.fwd(q, k, v, bias, mask + ci)
    assert _rel(out2, out0) < 1e-13


def test_backward_invariants_and_masking():
    B, N, H, d = 2, 9, 2, 4
    q, k, v, do, bias, mask = _rand(15, B, N, H, d, "ragged")
    dq, dk, dv, db = O.bwd(q, k, v, bias, mask, do)
    # every dbias row sums to zero over keys (sum_k ds_jk = 0 for each problem)
    np.testing.assert_allclose(db.sum(-1), 0.0, atol=1e-12)
    # masked keys: no gradient reaches them, exactly
    Lmask = mask.numpy() < -1e8
    for b in range(B):
        km = Lmask[b, 0]
        assert np.all(dk[b][:, km] == 0.0) and np.all(dv[b][:, km] == 0.0)
        assert np.all(db[b][:, :, km] == 0.0)
    # row subsets agree bitwise with the full computation
    rows = [(1, 3), (0, 0), (1, 8)]
    dq2, dk2, dv2 = O.bwd_rows(q, k, v, bias, mask, do, rows=rows)
    for (b, i) in rows:
        assert np.array_equal(dq2[b, i], dq[b, i]) and np.array_equal(dk2[b, i], dk[b, i])
        assert np.array_equal(dv2[b, i], dv[b, i])
    sel = [(1, 0, 4), (0, 1, 8)]
    db2 = O.dbias(q, k, v, bias, mask, do, sel=sel)
    for (b, h, j) in sel:
        assert np.array_equal(db2[b, h, j], db[b, h, j])
    out2, lse2 = O.fwd(q, k, v, bias, mask, rows=rows)
    out, lse = O.fwd(q, k, v, bias, mask)
    for (b, i) in rows:
        assert np.array_equal(out2[b, i], out[b, i]) and np.array_equal(lse2[b, :, i], lse[b, :, i])


def _fd_grads(q, k, v, bias, mask, do, eps=1e-6):
    def loss(q_, k_, v_, b_):
        out, _ = O.fwd(q_, k_, v_, b_, mask)
        return float((out * do.numpy()).sum())
    grads = []
    args = [q.numpy().copy(), k.numpy().copy(), v.numpy().copy(), bias.numpy().copy()]
    for a in range(4):
        g = np.zeros_like(args[a])
        it = np.nditer(args[a], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = args[a][idx]
            args[a][idx] = old + eps
            lp = loss(*args)
            args[a][idx] = old - eps
            lm = loss(*args)
            args[a][idx] = old
            g[idx] = (lp - lm) / (2 * eps)
        grads.append(g)
    return grads


@pytest.mark.parametrize("mk", ["none", "random"])
def test_gradients_match_central_finite_differences(mk):
    B, N, H, d = 1, 4, 2, 3
    q, k, v, do, bias, mask = _rand(16, B, N, H, d, mk)
    fd = _fd_grads(q, k, v, bias, mask, do)
    an = O.bwd(q, k, v, bias, mask, do)
    for g_fd, g_an in zip(fd, an):
        assert _rel(g_an, g_fd) < 1e-6


def test_ending_node_is_swapped_starting_node():
    B, N, H, d = 1, 6, 2, 4
    q, k, v, do, bias, mask = _rand(17, B, N, H, d, "random")
    out_e, lse_e = O.ending_fwd(q, k, v, bias, mask)
    # library path on the transposed pair tensors
    sw = lambda x: x.transpose(1, 2)
    ref = sw(_sdpa(sw(q), sw(k), sw(v), bias, mask, 1.0 / np.sqrt(d))).numpy()
    assert _rel(out_e, ref) < 1e-12
    dq, dk, dv, db = O.ending_bwd(q, k, v, bias, mask, do)
    qt, kt, vt, bt = (x.clone().requires_grad_(True) for x in (q, k, v, bias))
    o = sw(_sdpa(sw(qt), sw(kt), sw(vt), bt, mask, 1.0 / np.sqrt(d)))
    (o * do).sum().backward()
    for a, t in zip((dq, dk, dv, db), (qt, kt, vt, bt)):
        assert _rel(a, t.grad.numpy()) < 1e-11


def test_fully_masked_row_is_rejected():
    B, N, H, d = 1, 4, 1, 2
    q, k, v, do, bias, _ = _rand(18, B, N, H, d)
    mask = torch.zeros(B, N, N, dtype=torch.float64)
    mask[0, 2, :] = -1e9
    with pytest.raises(O.OracleError):
        O.fwd(q, k, v, bias, mask)


def _pins_pass(planted):
    """A compact run of the pins above with one planted mistake; True if all pass."""
    B, N, H, d = 2, 5, 2, 3
    q, k, v, do, bias, mask = _rand(19, B, N, H, d, "random")
    scale = 1.0 / np.sqrt(d)
    try:
        out, _ = O.fwd(q, k, v, bias, mask, scale, planted=planted)
        if _rel(out, _sdpa(q, k, v, bias, mask, scale).numpy()) > 1e-12:
            return False
        qt, kt, vt, bt = (x.clone().requires_grad_(True) for x in (q, k, v, bias))
        (_sdpa(qt, kt, vt, bt, mask, scale) * do).sum().backward()
        got = O.bwd(q, k, v, bias, mask, do, scale, planted=planted)
        for a, t in zip(got, (qt, kt, vt, bt)):
            if _rel(a, t.grad.numpy()) > 1e-11:
                return False
    except O.OracleError:
        return False
    return True


def test_pins_pass_on_the_unmodified_oracle():
    assert _pins_pass(0)


@pytest.mark.parametrize("planted", [1, 2, 3, 4, 5, 6, 7])
def test_pins_catch_planted_mistakes(planted):
    assert not _pins_pass(planted)


@pytest.mark.parametrize("mk", ["none", "ragged"])
def test_row_functions_equal_the_whole_stack(mk):
    """``row`` and ``dbias_streamed`` (one pair row at a time, for crops whose
    FP64 pair stack does not fit the host) run the whole-stack arithmetic on
    that row: bitwise equal to ``fwd``/``bwd_rows``/``dbias``, and pinned to
    the library attention as well."""
    q, k, v, do, bias, mask = _rand(41, 2, 11, 2, 4, mk)
    out, lse = O.fwd(q, k, v, bias, mask)
    dq, dk, dv = O.bwd_rows(q, k, v, bias, mask, do)
    db = O.dbias(q, k, v, bias, mask, do)
    ref_out = _sdpa(q, k, v, bias, mask, 0.5).numpy()
    for b, i in [(0, 0), (1, 7), (1, 10)]:
        m = None if mask is None else mask[b, i]
        o_r, l_r, dq_r, dk_r, dv_r = O.row(q[b, i], k[b, i], v[b, i], bias[b], m, do[b, i])
        assert np.array_equal(o_r, out[b, i]) and np.array_equal(l_r, lse[b, :, i])
        assert np.array_equal(dq_r, dq[b, i]) and np.array_equal(dk_r, dk[b, i]) and np.array_equal(dv_r, dv[b, i])
        assert _rel(o_r, ref_out[b, i]) < 1e-12
        o_f, l_f = O.row(q[b, i], k[b, i], v[b, i], bias[b], m)  # forward only
        assert np.array_equal(o_f, o_r) and np.array_equal(l_f, l_r)
    for b, h, j in [(0, 0, 0), (1, 1, 10), (0, 1, 5)]:
        get = lambda i: (q[b, i], k[b, i], v[b, i], None if mask is None else mask[b, i], do[b, i])
        assert np.array_equal(O.dbias_streamed(get, bias[b], h, j), db[b, h, j])
    for b in range(2):  # every (h, j) at once, one row at a time
        acc = np.zeros((2, 11, 11))
        for i in range(11):
            O.dbias_add_row(acc, q[b, i], k[b, i], v[b, i], bias[b], None if mask is None else mask[b, i], do[b, i])
        assert np.array_equal(acc, db[b])


def _literal_loops(q, k, v, bias, mask, do, scale):
    """The definition written out as plain Python loops over scalars (no array
    arithmetic), for tiny sizes: forward out and lse, then dv, dp, D, ds, dq, dk
    and dbias = sum over i of ds.  Shares nothing with the C oracle."""
    import math
    B, N, _, H, d = q.shape
    q, k, v, bias, do = (x.tolist() for x in (q, k, v, bias, do))
    mask = None if mask is None else mask.tolist()
    out = [[[[[0.0] * d for _ in range(H)] for _ in range(N)] for _ in range(N)] for _ in range(B)]
    lse = [[[[0.0] * N for _ in range(N)] for _ in range(H)] for _ in range(B)]
    dq = [[[[[0.0] * d for _ in range(H)] for _ in range(N)] for _ in range(N)] for _ in range(B)]
    dk = [[[[[0.0] * d for _ in range(H)] for _ in range(N)] for _ in range(N)] for _ in range(B)]
    dv = [[[[[0.0] * d for _ in range(H)] for _ in range(N)] for _ in range(N)] for _ in range(B)]
    db = [[[[0.0] * N for _ in range(N)] for _ in range(H)] for _ in range(B)]
    for b in range(B):
        for i in range(N):
            for h in range(H):
                p = [[0.0] * N for _ in range(N)]
                for j in range(N):
                    s = []
                    for kk in range(N):
                        dot = 0.0
                        for c in range(d):
                            dot += q[b][i][j][h][c] * k[b][i][kk][h][c]
                        x = scale * dot + bias[b][h][j][kk]
                        if mask is not None:
                            x += mask[b][i][kk]
                        s.append(x)
                    m = max(s)
                    z = 0.0
                    for kk in range(N):
                        z += math.exp(s[kk] - m)
                    lse[b][h][i][j] = m + math.log(z)
                    for kk in range(N):
                        p[j][kk] = math.exp(s[kk] - m) / z
                    for c in range(d):
                        acc = 0.0
                        for kk in range(N):
                            acc += p[j][kk] * v[b][i][kk][h][c]
                        out[b][i][j][h][c] = acc
                for j in range(N):
                    Dj = 0.0
                    for c in range(d):
                        Dj += do[b][i][j][h][c] * out[b][i][j][h][c]
                    for kk in range(N):
                        dp = 0.0
                        for c in range(d):
                            dp += do[b][i][j][h][c] * v[b][i][kk][h][c]
                        ds = p[j][kk] * (dp - Dj)
                        db[b][h][j][kk] += ds
                        for c in range(d):
                            dv[b][i][kk][h][c] += p[j][kk] * do[b][i][j][h][c]
                            dq[b][i][j][h][c] += scale * ds * k[b][i][kk][h][c]
                            dk[b][i][kk][h][c] += scale * ds * q[b][i][j][h][c]
    return tuple(np.array(x) for x in (out, lse, dq, dk, dv, db))


@pytest.mark.parametrize("N,mk", [(2, "none"), (3, "random"), (5, "ragged"), (8, "random")])
def test_oracle_equals_literal_loops_on_tiny_sizes(N, mk):
    """Brute force: the definition as scalar Python loops agrees with the C oracle
    to 1e-12 on tiny pair stacks (H=2, d=4), forward and all four gradients."""
    q, k, v, do, bias, mask = _rand(40 + N, 2 if N < 8 else 1, N, 2, 4, mk)
    scale = 1.0 / np.sqrt(4)
    out_l, lse_l, dq_l, dk_l, dv_l, db_l = _literal_loops(q.numpy(), k.numpy(), v.numpy(), bias.numpy(),
                                                         None if mask is None else mask.numpy(), do.numpy(), scale)
    out, lse = O.fwd(q, k, v, bias, mask, scale)
    dq, dk, dv, db = O.bwd(q, k, v, bias, mask, do, scale)
    for got, ref in ((out, out_l), (lse, lse_l), (dq, dq_l), (dk, dk_l), (dv, dv_l), (db, db_l)):
        assert _rel(got, ref) < 1e-12


@pytest.mark.parametrize("planted", [1, 2, 3, 4, 5, 6, 7])
def test_literal_loops_catch_planted_mistakes(planted):
    """The brute-force pin on its own also catches every planted mistake."""
    N = 5
    q, k, v, do, bias, mask = _rand(45, 1, N, 2, 3, "random")
    scale = 1.0 / np.sqrt(3)
    ref = _literal_loops(q.numpy(), k.numpy(), v.numpy(), bias.numpy(), mask.numpy(), do.numpy(), scale)
    try:
        out, lse = O.fwd(q, k, v, bias, mask, scale, planted=planted)
        got = (out, lse) + tuple(O.bwd(q, k, v, bias, mask, do, scale, planted=planted))
    except O.OracleError:
        return
    assert max(_rel(g, r) for g, r in zip(got, ref)) > 1e-12
