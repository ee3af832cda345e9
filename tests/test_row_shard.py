"""Row-sharded path (rows i split across ranks, dBias exchanged; row_shard.py).

CPU (no GPU): the row partition, and the dBias exchange of two and three gloo ranks
whose shares come from the FP64 oracle -- a rank's share of the sum over rows i is
the oracle's dBias with dout zeroed outside the rank's rows, since a row with zero
upstream gradient has zero score gradient.
GPU: shards run one after another on one device against the whole problem (o,
resid, lse, dq, dk, dv bit for bit; dBias against the oracle and repeatable), and
the NCCL code path of shard_bwd with a single rank.  Runs of several GPUs whose
kernels wait on one another are not emulated on one device.
"""
import os
import socket

import numpy as np
import pytest
import torch

from triangle_attention_biomolecular_b200 import row_shard as RS


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("N", [1, 2, 7, 8, 200, 768, 769])
def test_row_range_partitions_the_rows(N):
    for world in range(1, min(N, 9) + 1):
        blocks = [RS.row_range(N, r, world) for r in range(world)]
        assert blocks[0][0] == 0
        for (i0, n0), (i1, _) in zip(blocks, blocks[1:]):
            assert i1 == i0 + n0  # contiguous, in rank order
        assert sum(n for _, n in blocks) == N
        sizes = [n for _, n in blocks]
        assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        RS.row_range(N, 0, N + 1)
    with pytest.raises(ValueError):
        RS.row_range(N, 1, 1)


def test_partial_slots_are_the_most_any_block_needs():
    from triangle_attention_biomolecular_b200 import _binding as Bd
    # N=80 over 9 ranks: blocks of 9 rows take two partials, the block of 8 takes one
    per_rank = [Bd.tri_attn_bwd_rows_dbias_parts(1, RS.row_range(80, r, 9)[1], 80, 4, 32) for r in range(9)]
    assert per_rank == [2] * 8 + [1]
    assert RS.dbias_parts(1, 80, 4, 32, 9) == 2
    assert RS.dbias_parts(1, 768, 4, 32, 2) == 1  # crop768: no row chunks


def _wrong_parts_worker(rank, port):
    import torch.distributed as dist
    from triangle_attention_biomolecular_b200 import _binding as Bd
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=1)
    try:
        q = torch.zeros((1, 16, 16, 2, 32), dtype=torch.bfloat16)
        parts = torch.zeros((5, 1, 2, 16, 16))  # the right count is 2
        with pytest.raises(Bd.TriAttnError):
            RS.shard_bwd(q, q, q, None, None, q, q, None, q, q, q, q, None, None, parts)
    finally:
        dist.destroy_process_group()


def test_shard_bwd_checks_the_partials_buffer_first():
    import torch.multiprocessing as mp
    mp.spawn(_wrong_parts_worker, args=(free_port(),), nprocs=1, join=True)


def small_problem(seed=3, B=1, N=10, H=2, d=8):
    g = torch.Generator().manual_seed(seed)
    q, k, v, dout = (torch.randn((B, N, N, H, d), generator=g).to(torch.bfloat16) for _ in range(4))
    bias = torch.randn((B, H, N, N), generator=g).to(torch.bfloat16)
    mask = torch.zeros((B, N, N))
    mask[:, :, N - 2:] = -1e9  # the last two keys padded
    return q, k, v, bias, mask, dout


def _exchange_worker(rank, world, port, tmpdir):
    import torch.distributed as dist
    from oracle import oracle as O
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, bias, mask, dout = small_problem()
        N = q.shape[1]
        i0, rows = RS.row_range(N, rank, world)
        mine = torch.zeros_like(dout)
        mine[:, i0:i0 + rows] = dout[:, i0:i0 + rows]
        part = O.dbias(q, k, v, bias, mask, mine)                        # this rank's share, FP64
        local = torch.from_numpy(part).float().unsqueeze(0)              # [1,B,H,N,N] FP32
        gathered = RS.gather_parts(local)
        assert tuple(gathered.shape) == (world,) + tuple(local.shape[1:])
        assert torch.equal(gathered[rank], local[0])                     # own share in its rank slot
        total = gathered[0].clone()
        for p in range(1, world):                                        # ascending rank order
            total += gathered[p]
        np.save(os.path.join(tmpdir, f"total{rank}.npy"), total.numpy())
        np.save(os.path.join(tmpdir, f"gathered{rank}.npy"), gathered.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_dbias_exchange_matches_the_whole_sum(world, tmp_path):
    import torch.multiprocessing as mp
    from oracle import oracle as O
    O.build()
    mp.spawn(_exchange_worker, args=(world, free_port(), str(tmp_path)), nprocs=world, join=True)
    totals = [np.load(tmp_path / f"total{r}.npy") for r in range(world)]
    gathered = [np.load(tmp_path / f"gathered{r}.npy") for r in range(world)]
    for r in range(1, world):
        assert np.array_equal(gathered[r], gathered[0])                  # every rank sees the same array
        assert np.array_equal(totals[r], totals[0])                      # ... and the same bits
    q, k, v, bias, mask, dout = small_problem()
    whole = O.dbias(q, k, v, bias, mask, dout)
    np.testing.assert_allclose(totals[0], whole, rtol=1e-5, atol=1e-6)  # FP32 rounding of the shares


# ------------------------------------------------------------------------- GPU

def _views(t, i0, rows):
    return t[:, i0:i0 + rows]


def run_shards(x, world, dev):
    from triangle_attention_biomolecular_b200 import _binding as Bd
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "dout"))
    bias = x["bias"].to(dev)
    mask = x["mask"].to(dev) if x["mask"] is not None else None
    B, N, _, H, d = q.shape
    o, r = torch.empty_like(q), torch.empty_like(q)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    lses, parts = [], []
    P = RS.dbias_parts(B, N, H, d, world)
    for rank in range(world):
        i0, rows = RS.row_range(N, rank, world)
        sl = lambda t: _views(t, i0, rows)
        m = sl(mask) if mask is not None else None
        lse = torch.empty((B, H, rows, N), dtype=torch.float32, device=dev)
        Bd.tri_attn_fwd_rows(sl(q), sl(k), sl(v), bias, m, sl(o), sl(r), lse)
        ws = torch.empty(Bd.tri_attn_bwd_rows_workspace_bytes(B, rows, N, H, d), dtype=torch.uint8, device=dev)
        pr = torch.zeros((P, B, H, N, N), dtype=torch.float32, device=dev)
        mine = Bd.tri_attn_bwd_rows_dbias_parts(B, rows, N, H, d)
        Bd.tri_attn_bwd_rows(sl(q), sl(k), sl(v), bias, m, sl(o), sl(r), lse, sl(do), sl(dq), sl(dk), sl(dv),
                             pr[:mine], ws)
        lses.append(lse)
        parts.append(pr)
    db = torch.empty((B, H, N, N), dtype=torch.bfloat16, device=dev)
    Bd.tri_attn_dbias_sum(torch.cat(parts), db)
    torch.cuda.synchronize()
    st, word = Bd.tri_attn_device_error(True)
    assert st == Bd.TRI_ATTN_OK, f"device error word {word:#x}"
    return {"out": o, "resid": r, "lse": torch.cat(lses, dim=2), "dq": dq, "dk": dk, "dv": dv, "dbias": db}


@pytest.mark.gpu
# (80, 9): blocks of 9 rows take two dBias partials, the block of 8 one, so the
# padded (zero) slot of the exchange is exercised
@pytest.mark.parametrize("N,world,d", [(200, 2, 32), (200, 3, 64), (384, 3, 32), (144, 5, 32), (80, 9, 32)])
def test_shards_match_the_whole_problem(N, world, d):
    from oracle import oracle as O
    from triangle_attention_biomolecular_b200 import api
    from triangle_attention_biomolecular_b200 import synthetic as S
    wl = S.Workload(f"shard N={N}", 1, N, 4, d, mask="ragged", len_lo=N * 3 // 4, len_hi=N)
    x = S.make_inputs(wl, 11 + N + world)
    dev = torch.device("cuda")
    got = run_shards(x, world, dev)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "dout"))
    bias, mask = x["bias"].to(dev), x["mask"].to(dev)
    o, r, lse = api.forward(q, k, v, bias, mask)
    dq, dk, dv, db = api.backward(q, k, v, bias, mask, o, r, lse, do)
    torch.cuda.synchronize()
    whole = {"out": o, "resid": r, "lse": lse, "dq": dq, "dk": dk, "dv": dv}
    for n, t in whole.items():  # per-row problems: the same arithmetic, bit for bit
        assert torch.equal(got[n], t), n
    # dBias: the shares add up in another order than the whole problem's chunks
    ref = O.dbias(x["q"], x["k"], x["v"], x["bias"], x["mask"], x["dout"])
    g64 = got["dbias"].double().cpu().numpy()
    err = float(np.linalg.norm(g64 - ref) / np.linalg.norm(ref))
    assert err <= 2e-2, err
    diff = (got["dbias"].float() - db.float()).abs().max().item()
    assert diff <= 2e-2 * db.float().abs().max().item(), diff
    again = run_shards(x, world, dev)
    assert torch.equal(again["dbias"], got["dbias"])  # fixed order: repeatable bit for bit


@pytest.mark.gpu
def test_crop768_two_shards_against_the_whole_problem():
    # the headline size: one dBias partial per block (no row chunks); the whole problem's
    # own dBias, already within the oracle gate (test_gpu_parity), is the reference
    from triangle_attention_biomolecular_b200 import api
    from triangle_attention_biomolecular_b200 import synthetic as S
    x = S.make_inputs(S.CROP768, 41)
    dev = torch.device("cuda")
    got = run_shards(x, 2, dev)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "dout"))
    bias, mask = x["bias"].to(dev), x["mask"].to(dev)
    o, r, lse = api.forward(q, k, v, bias, mask)
    dq, dk, dv, db = api.backward(q, k, v, bias, mask, o, r, lse, do)
    torch.cuda.synchronize()
    for n, t in {"out": o, "resid": r, "lse": lse, "dq": dq, "dk": dk, "dv": dv}.items():
        assert torch.equal(got[n], t), n
    a, b = got["dbias"].double(), db.double()
    assert float((a - b).norm() / b.norm()) < 2e-3  # two FP32 partials vs one sum: BF16-level differences


def _nccl_one_rank(rank, port):
    import torch.distributed as dist
    from triangle_attention_biomolecular_b200 import _binding as Bd
    from triangle_attention_biomolecular_b200 import api
    from triangle_attention_biomolecular_b200 import synthetic as S
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        wl = S.Workload("nccl one rank", 1, 160, 4, 32, mask="ragged", len_lo=120, len_hi=160)
        x = S.make_inputs(wl, 5)
        q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "dout"))
        bias, mask = x["bias"].to(dev), x["mask"].to(dev)
        B, N, _, H, d = q.shape
        i0, rows = RS.row_range(N, 0, 1)
        o, r = torch.empty_like(q), torch.empty_like(q)
        lse = torch.empty((B, H, rows, N), dtype=torch.float32, device=dev)
        RS.shard_fwd(q, k, v, bias, mask, o, r, lse)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        db = torch.empty((B, H, N, N), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(Bd.tri_attn_bwd_rows_workspace_bytes(B, rows, N, H, d), dtype=torch.uint8, device=dev)
        parts = torch.empty((RS.dbias_parts(B, N, H, d, 1), B, H, N, N), dtype=torch.float32, device=dev)
        RS.shard_bwd(q, k, v, bias, mask, o, r, lse, do, dq, dk, dv, db, ws, parts)
        o2, r2, lse2 = api.forward(q, k, v, bias, mask)
        dq2, dk2, dv2, db2 = api.backward(q, k, v, bias, mask, o2, r2, lse2, do)
        torch.cuda.synchronize()
        for a, b in ((o, o2), (r, r2), (lse, lse2), (dq, dq2), (dk, dk2), (dv, dv2)):
            assert torch.equal(a, b)
        # one rank: the same partial sums in the same order as the whole problem's chunks
        assert torch.equal(db, db2)
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_nccl_path_with_one_rank():
    import torch.multiprocessing as mp
    mp.spawn(_nccl_one_rank, args=(free_port(),), nprocs=1, join=True)
