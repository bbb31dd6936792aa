"""The row-sharded update's bookkeeping on CPU (no GPU): shard boundaries, which operand is
exchanged, which of a's columns the incoming contraction reads, and the assembly of the
shards' rows, with two gloo ranks.

Each rank runs the two phases with fp64 stand-ins written from the oracle's steps (the
gated projection of its rows; the contraction of its rows from the exchanged planes, then the
output gate); the exchange is RowShardedTriMul's own all-gather. The rows put together must
equal the oracle's update of the whole pair tensor."""
import ctypes
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from protein_pair_representation_b200 import trimul as tm


def test_shard_bounds():
    assert tm.shard_bounds(256, 2) == [0, 128, 256]
    assert tm.shard_bounds(640, 3) == [0, 256, 512, 640]
    assert tm.shard_bounds(2048, 8) == [0, 256, 512, 768, 1024, 1280, 1536, 1792, 2048]
    assert tm.shard_bounds(128, 1) == [0, 128]
    for N, G in ((100, 1), (256, 3), (256, 0)):
        with pytest.raises(ValueError):
            tm.shard_bounds(N, G)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _phases(inp):
    import oracle
    W = inp.weights

    def project(z_rows, mask_rows, row0, N):
        zh = oracle.layernorm(z_rows.numpy(), W["ln_in_g"], W["ln_in_b"], inp.eps)
        m = mask_rows.numpy()
        a = oracle.gated_projection(zh, m, W["w_ag"], W["b_ag"], W["w_ap"], W["b_ap"])
        b = oracle.gated_projection(zh, m, W["w_bg"], W["b_bg"], W["w_bp"], W["b_bp"])
        # the library's layout: [B, c_h, R, N]
        return torch.from_numpy(np.ascontiguousarray(a.transpose(0, 3, 1, 2))), \
            torch.from_numpy(np.ascontiguousarray(b.transpose(0, 3, 1, 2)))

    def finish(z_rows, mask_rows, row0, N, direction, bounds, a_all, b_all, out=None):
        rank = bounds.index(row0)
        R = bounds[rank + 1] - row0
        b_full = torch.cat(b_all, dim=2).numpy()                     # [B, c, N (rows j or k), N]
        if direction == "outgoing":
            assert all(a is None for g, a in enumerate(a_all) if g != rank)
            x = np.einsum("bcik,bcjk->bcij", a_all[rank].numpy(), b_full)
        else:
            a_full = torch.cat(a_all, dim=2).numpy()                 # rows k of every shard
            x = np.einsum("bcki,bckj->bcij", a_full[:, :, :, row0:row0 + R], b_full)
        zh = oracle.layernorm(z_rows.numpy(), W["ln_in_g"], W["ln_in_b"], inp.eps)
        o = oracle.output_gate(zh, x.transpose(0, 2, 3, 1), mask_rows.numpy(), W["w_g"], W["b_g"], W["ln_out_g"],
                               W["ln_out_b"], inp.eps, W["w_o"], W["b_o"])
        return torch.from_numpy(o)

    return project, finish


def _worker(rank, world, port, N, bounds_in, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import trimul_inputs as ti
        from protein_pair_representation_b200.sharded import RowShardedTriMul
        inp = ti.generate(2, N, 16, 8, dtype="f32", seed=9, mask=("uniform_len", N // 2, N), affine=True,
                          biases=True)
        project, finish = _phases(inp)
        sh = RowShardedTriMul(project=project, finish=finish)
        bounds = sh.bounds(N)
        assert bounds == bounds_in
        r0, r1 = bounds[rank], bounds[rank + 1]
        z = torch.from_numpy(inp.z[:, r0:r1].astype(np.float64))
        m = torch.from_numpy(inp.mask[:, r0:r1].astype(np.float64))
        for d in ("outgoing", "incoming"):
            rows = sh(z, m, N, d)
            q.put((rank, d, r0, rows.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("N,world", [(256, 2), (384, 2)])
def test_two_gloo_ranks_assemble_the_oracle_update(N, world):
    import oracle
    import trimul_inputs as ti
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    bounds = tm.shard_bounds(N, world)
    procs = [ctx.Process(target=_worker, args=(r, world, port, N, bounds, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=300) for _ in range(2 * world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    inp = ti.generate(2, N, 16, 8, dtype="f32", seed=9, mask=("uniform_len", N // 2, N), affine=True, biases=True)
    for d in ("outgoing", "incoming"):
        rows = sorted((r0, x) for rank, dd, r0, x in got if dd == d)
        full = np.concatenate([x for _, x in rows], axis=1)
        ref = oracle.trimul(inp.z, inp.mask, inp.weights, d, inp.eps)
        assert np.max(np.abs(full - ref)) <= 1e-12 * np.max(np.abs(ref)), d
        # and the exchange mattered: a rank's rows differ from what its rows alone would give
        assert full.shape == ref.shape


def test_shard_entry_points_validate_on_the_host():
    """Size and shard-table rules are answered before the layer and any device call."""
    lib = tm.load_library()
    def rows(data, B, R, N, C, row0, dtype=tm.BF16):
        return tm._Rows(data, B, R, N, C, row0, dtype)
    fake = 1 << 24
    z = rows(fake, 1, 128, 200, 128, 0)                           # N not a multiple of 128
    assert lib.tri_mul_shard_project(ctypes.byref(z), None, None, fake << 4, fake << 5, None) == 2
    z = rows(fake, 1, 100, 256, 128, 0)                           # rows not whole 128-row blocks
    assert lib.tri_mul_shard_project(ctypes.byref(z), None, None, fake << 4, fake << 5, None) == 2
    z = rows(fake, 1, 128, 256, 128, 0, tm.F32)                   # tensor-core path only
    assert lib.tri_mul_shard_project(ctypes.byref(z), None, None, fake << 4, fake << 5, None) == 2
    z = rows(fake, 1, 128, 256, 128, 128)
    assert lib.tri_mul_shard_project(ctypes.byref(z), None, None, fake << 4, fake << 5, None) == 1
    assert b"layer is NULL" in lib.tri_mul_last_error()
    out = rows(fake << 8, 1, 128, 256, 128, 128, tm.F32)
    table = (ctypes.c_int64 * 3)(0, 128, 256)
    ptrs = (ctypes.c_void_p * 2)(fake << 4, fake << 5)
    assert lib.tri_mul_shard_finish(ctypes.byref(z), None, None, 0, 9, table, ptrs, ptrs, ctypes.byref(out), None) == 2
    assert lib.tri_mul_shard_finish(ctypes.byref(z), None, None, 0, 2, table, ptrs, ptrs, ctypes.byref(out), None) == 1
    assert b"layer is NULL" in lib.tri_mul_last_error()
    bad = (ctypes.c_int64 * 3)(0, 128, 200)
    assert lib.tri_mul_shard_finish(ctypes.byref(z), None, None, 0, 2, bad, ptrs, ptrs, ctypes.byref(out), None) == 1
    other = rows(fake, 1, 128, 256, 128, 64)                       # starts inside a block
    assert lib.tri_mul_shard_finish(ctypes.byref(other), None, None, 0, 2, table, ptrs, ptrs, ctypes.byref(out), None) == 2
