"""Multi-rank host logic on CPU: world-size-2 gloo process groups, no GPU.

The data path has no collective (chains are independent); these tests cover what the ranks do
share: the partition of a packed batch, the head split and the max/sum reductions of timings.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp

from gated_delta_rule_144_b200 import shard, synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import json

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lengths = synth.doc_lengths(8, 512, 8192, 32768, seed=1002)
        parts = shard.partition_documents(lengths, world)
        gathered = [None] * world
        dist.all_gather_object(gathered, parts)
        heads = shard.split_heads(32, world)
        t_max = shard.max_over_ranks(1.5 + rank)        # ranks report 1.5 and 2.5
        t_sum = shard.sum_over_ranks(10.0 * (rank + 1))  # 10 + 20
        shard.barrier()
        res = {"rank": rank, "parts": parts, "gathered": gathered,
               "heads": [[h.start, h.stop] for h in heads], "max": t_max, "sum": t_sum,
               "lengths": lengths}
        with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as fh:
            json.dump(res, fh)
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_ranks(tmp_path_factory):
    import json
    out = tmp_path_factory.mktemp("ranks")
    mp.start_processes(_worker, args=(2, _free_port(), str(out)), nprocs=2, join=True,
                       start_method="spawn")
    return [json.load(open(out / ("rank%d.json" % r))) for r in range(2)]


def test_ranks_agree_on_the_document_partition(two_ranks):
    a, b = two_ranks
    assert a["parts"] == b["parts"]
    assert a["gathered"][0] == a["gathered"][1] == a["parts"]


def test_partition_covers_every_document_once(two_ranks):
    parts, lengths = two_ranks[0]["parts"], two_ranks[0]["lengths"]
    flat = sorted(i for p in parts for i in p)
    assert flat == list(range(len(lengths)))
    loads = [sum(lengths[i] for i in p) for p in parts]
    # longest-processing-time bound: makespan <= 4/3 of the optimum >= max(mean, longest doc)
    lower = max(sum(lengths) / 2, max(lengths))
    assert max(loads) <= 4 / 3 * lower + 1


def test_heads_split_evenly(two_ranks):
    assert two_ranks[0]["heads"] == [[0, 16], [16, 32]]


def test_timing_reductions(two_ranks):
    for r in two_ranks:
        assert r["max"] == 2.5
        assert r["sum"] == 30.0


def test_single_process_helpers_without_a_group():
    assert shard.max_over_ranks(3.0) == 3.0
    assert shard.sum_over_ranks(4.0) == 4.0
    assert [len(h) for h in shard.split_heads(7, 3)] == [3, 2, 2]
    assert shard.partition_documents([5, 0, 3], 4) == [[0], [2], [1], []]
    assert shard.rank_seed(1004, 0) != shard.rank_seed(1004, 1)
