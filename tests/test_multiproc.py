"""Row-sharded codec on two ranks (gloo, CPU): each rank encodes its own row
block with no communication; an all-gather of word counts rebases the
offsets; the stitched stream equals a single encode of the whole matrix bit
for bit.  The per-rank encode is the oracle here (the kernels need a GPU);
what is tested is the host-side sharding logic of the package."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROWS, COLS, TILE, LAT, BPS, SEED = 37, 768, 256, "E8", 4.0, 11


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _matrix():
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(ROWS, COLS, generator=g) * 0.02).to(torch.bfloat16)
    return x.view(torch.int16).numpy().view(np.uint16)


def _worker(rank, world, port, outdir):
    import oracle
    from kv_quantization_tile_b200 import sharding

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        x = _matrix()
        r0, r1 = sharding.row_range(ROWS, rank, world)
        local = oracle.encode(x[r0:r1], TILE, LAT, BPS, SEED)
        base, total = sharding.global_word_base(int(local["off"][-1]))
        off = sharding.rebase_offsets(torch.from_numpy(local["off"].astype(np.int64)), base,
                                      rank == world - 1)
        # gather everything on every rank to stitch and check
        parts = [None] * world
        dist.all_gather_object(parts, {"off": off.numpy(), "payload": local["payload"],
                                       "scale": local["scale"], "k": local["k"], "base": base,
                                       "total": total})
        if rank == 0:
            stitched = {"off": np.concatenate([p["off"] for p in parts]).astype(np.uint32),
                        "payload": np.concatenate([p["payload"] for p in parts]),
                        "scale": np.concatenate([p["scale"] for p in parts]),
                        "k": np.concatenate([p["k"] for p in parts])}
            np.savez(os.path.join(outdir, "stitched.npz"), **stitched)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world", [2])
def test_row_sharded_stream_equals_single_encode(tmp_path, world):
    import oracle
    from kv_quantization_tile_b200 import sharding

    assert [sharding.row_range(ROWS, r, world) for r in range(world)] == [(0, 19), (19, 37)]
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    got = np.load(os.path.join(tmp_path, "stitched.npz"))
    ref = oracle.encode(_matrix(), TILE, LAT, BPS, SEED)
    for key in ("off", "payload", "scale", "k"):
        assert np.array_equal(got[key], ref[key]), key


def test_row_range_covers_rows():
    from kv_quantization_tile_b200 import sharding
    for rows in (0, 1, 7, 100):
        for world in (1, 2, 3, 8):
            spans = [sharding.row_range(rows, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == rows
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            assert max(b - a for a, b in spans) - min(b - a for a, b in spans) <= 1
