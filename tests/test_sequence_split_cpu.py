"""Host logic of decoding a sequence whose cache is split over ranks by token range,
on CPU: the token ranges, the per-range lengths, and the exchange step of
``SplitSequenceDecoder`` run by two gloo ranks. Each rank fills its partial with the
oracle's decode of its own range; after the all-gather every rank merges the parts
(with the oracle's merge) and must get the oracle's decode over the whole cache."""
import json
import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
from kv_cache_vector_05_b200.sequence_split import SplitSequenceDecoder, local_lengths, token_range  # noqa: E402


@pytest.mark.parametrize("n,world,block", [(0, 2, 512), (1, 4, 512), (1500, 3, 512), (1 << 20, 8, 512),
                                           (4097, 2, 512), (10, 3, 4), (700, 5, 128)])
def test_token_ranges_tile_the_sequence(n, world, block):
    ranges = [token_range(n, world, r, block) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == n
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0                                      # contiguous, in rank order
    for a, b in ranges:
        assert 0 <= a <= b <= n and (a % block == 0 or a == n)  # ranges start on a block
    sizes = [-(-(b - a) // block) for a, b in ranges]        # blocks per rank
    assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)


def test_token_range_rejects_bad_arguments():
    for args in [(-1, 2, 0), (10, 0, 0), (10, 2, 2), (10, 2, -1)]:
        with pytest.raises(ValueError):
            token_range(*args)


def test_local_lengths():
    lens = torch.tensor([1500, 700, 0, 512], dtype=torch.int32)
    assert local_lengths(lens, 0, 512).tolist() == [512, 512, 0, 512]
    assert local_lengths(lens, 512, 1024).tolist() == [512, 188, 0, 0]
    assert local_lengths(lens, 1024, 1500).tolist() == [476, 0, 0, 0]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


D, G, BATCH, HKV, N_TOK, BLOCK, VB = 32, 2, 2, 1, 1100, 512, 2
LENS = [1100, 530]


def _cache():
    import oracle as O
    rng = np.random.default_rng(41)
    Pi = O.hadamard_rotation(np.where(rng.integers(0, 2, D) == 1, 1, -1))
    S = rng.standard_normal((D, D))
    c, t = O.device_codebook(D, 2)
    K = rng.standard_normal((BATCH, N_TOK, D))
    V = rng.standard_normal((BATCH, N_TOK, D))
    q = rng.standard_normal((BATCH, G, D))
    pk = [O.compress_keys(K[b], Pi, c, t, S) for b in range(BATCH)]
    pv = [O.quantize_values(V[b], VB) for b in range(BATCH)]
    return O, Pi, S, c, pk, pv, q


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        O, Pi, S, c, pk, pv, q = _cache()
        start, end = token_range(N_TOK, world, rank, BLOCK)
        lens = local_lengths(torch.tensor(LENS, dtype=torch.int32), start, end).tolist()
        dec = SplitSequenceDecoder(BATCH, G * HKV, D, device="cpu")
        assert (dec.world, dec.rank) == (world, rank)
        out, lse = dec.local_out(), dec.local_lse()
        for b in range(BATCH):                               # this rank's partial, by the oracle
            pk_r = {k: v[start:end] for k, v in pk[b].items()}
            pv_r = {k: v[start:end] for k, v in pv[b].items()}
            sc, o = O.decode_attention(q[b], pk_r, pv_r, Pi, c, S, D, VB, length=lens[b])
            out[b] = torch.from_numpy(o)
            lse[b] = torch.from_numpy(O.log_partition(sc, lens[b]))
        dec.exchange()
        outs, lses = dec.gathered_parts()
        mine_out, mine_lse = outs[rank].clone(), lses[rank].clone()
        res = {"own_part_in_place": bool(torch.equal(mine_out, out) and torch.equal(mine_lse, lse)), "rows": []}
        for b in range(BATCH):
            merged, _ = O.merge_attention(outs[:, b].double().numpy(), lses[:, b].double().numpy())
            _, whole = O.decode_attention(q[b], pk[b], pv[b], Pi, c, S, D, VB, length=LENS[b])
            res["rows"].append(float(np.abs(merged - whole).max()))
        res["lse_rank1"] = [float(lses[1, 0, 0]), float(lses[1, 1, 0])]
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_exchange_and_merge_to_the_whole_decode(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["own_part_in_place"]
        assert max(r["rows"]) < 1e-6                         # fp32 exchange of fp64 partials
        # rank 1 holds tokens [1024, 1100): 76 of sequence 0, none of sequence 1 (530 tokens),
        # whose empty range has lse = -inf and weighs nothing in the merge
        assert np.isfinite(r["lse_rank1"][0]) and r["lse_rank1"][1] == -np.inf
    assert res[0] == res[1]                                  # every rank gets the same result
