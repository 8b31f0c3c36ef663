"""Expert-parallel sharding (grouped_bit_weight_b200.ep) across gloo ranks
on CPU: the dispatch / combine plumbing around the per-rank grouped call.

Each rank owns E / world experts.  The local call is the CPU oracle's
grouped forward on the rows the rank received (the product passes the
library's kernels there; this file tests the exchange, not the kernels).
Because the oracle computes every routed row on its own, the expert-parallel
result must equal, bit for bit, the oracle's grouped forward of the rank's
own tokens against all E experts -- any row sent to the wrong rank, paired
with the wrong expert or put back in the wrong (token, slot) place breaks
that equality."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle as orc
import synth
from gpu_util import packed_weights

E, N, K, TOPK = 8, 24, 128, 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _to_t(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _topk(T: int, seed: int, k: int = TOPK, hot: int = -1) -> np.ndarray:
    """k distinct experts per token, uniform; hot >= 0 sends every token's
    first slot to expert `hot`."""
    rng = np.random.default_rng(seed)
    if not T:
        return np.zeros((0, k), np.int64)
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int64)
    if hot >= 0:
        for t in range(T):
            if hot in ids[t, 1:]:
                ids[t, list(ids[t]).index(hot)] = ids[t, 0]
            ids[t, 0] = hot
    return ids


def _reference(x_bits, ids, wdec):
    """The oracle's grouped forward of this rank's tokens over all experts,
    scattered to [T, k, N]."""
    T, k = ids.shape
    flat = ids.reshape(-1)
    order = np.argsort(flat, kind="stable")
    off = np.searchsorted(flat[order], np.arange(E + 1)).astype(np.int32)
    out = orc.grouped_forward(x_bits, wdec, off, (order // k).astype(np.int32))
    y = np.zeros((T * k, N), np.uint16)
    y[order] = out
    return y.reshape(T, k, N)


def _rank(rank, world, port, tokens, q, k=TOPK, hot=-1):
    import torch.distributed as dist

    from grouped_bit_weight_b200.ep import ExpertParallel
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wdec = packed_weights("nf4", E, N, K, 0.05, 41)[2]
        T = tokens[rank]
        x_bits = synth.to_bf16_bits(synth.normal((T, K), 100 + rank)) if T else \
            np.zeros((0, K), np.uint16)
        ids = _topk(T, 200 + rank, k, hot)
        ep = ExpertParallel(E)
        e0, e1 = ep.first_expert, ep.first_expert + ep.E_local
        seen = {}

        def local(xr, off, r2t):
            seen["rows"] = int(off[-1])
            seen["experts_ok"] = off.shape[0] == ep.E_local + 1
            out = orc.grouped_forward(_bits(xr), wdec[e0:e1], off.numpy(), r2t.numpy())
            return _to_t(out)

        y = ep.run(_to_t(x_bits), torch.from_numpy(ids), local)
        ref = _reference(x_bits, ids, wdec)

        # positive control: the same exchange with this rank's experts
        # listed in reverse order must give a different result somewhere
        def local_swapped(xr, off, r2t):
            out = orc.grouped_forward(_bits(xr), wdec[e0:e1][::-1].copy(), off.numpy(),
                                      r2t.numpy())
            return _to_t(out)
        y_bad = ep.run(_to_t(x_bits), torch.from_numpy(ids), local_swapped)
        all_bad = [None] * world
        dist.all_gather_object(all_bad, bool(np.array_equal(_bits(y_bad), ref)))
        # rows this rank's experts received = routed rows of all ranks to them
        sent_here = 0
        for r in range(world):
            ids_r = _topk(tokens[r], 200 + r, k, hot)
            sent_here += int(((ids_r >= e0) & (ids_r < e1)).sum())
        q.put((rank, bool(np.array_equal(_bits(y), ref)), tuple(y.shape),
               seen["rows"] == sent_here, seen["experts_ok"], not all(all_bad)))
    finally:
        dist.destroy_process_group()


def _launch(tokens, k=TOPK, hot=-1):
    world, port = len(tokens), _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, tokens, q, k, hot))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(world))
    for (rank, same, shape, rows_ok, experts_ok, control_caught), T in zip(got, tokens):
        assert shape == (T, k, N), (rank, shape)
        assert rows_ok and experts_ok, rank
        assert same, f"rank {rank}: expert-parallel output differs from the oracle"
        assert control_caught, "swapping a rank's experts went unnoticed"


def test_two_ranks_uneven_token_counts():
    _launch([5, 33])


def test_four_ranks_with_an_idle_rank():
    """Rank 2 has no tokens (it still serves its two experts)."""
    _launch([7, 19, 0, 12])


def test_two_ranks_top1_routing():
    _launch([6, 17], k=1)


def test_every_token_sends_its_first_slot_to_one_expert():
    """Expert 7 (the last rank's) receives a row from every token of every
    rank; the other slots stay uniform."""
    _launch([9, 4], k=3, hot=7)


def test_single_rank_holds_every_expert_and_rejects_bad_ids():
    import torch.distributed as dist

    from grouped_bit_weight_b200.ep import ExpertParallel
    port = _free_port()
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=30))
    try:
        ep = ExpertParallel(3)  # one rank holds all three
        assert (ep.E_local, ep.first_expert) == (3, 0)
        with pytest.raises(ValueError):
            ep.dispatch(torch.zeros((2, K), dtype=torch.bfloat16), torch.tensor([[0, 3], [1, 2]]))
    finally:
        dist.destroy_process_group()
