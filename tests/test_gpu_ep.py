"""ep_grouped_gemm on one GPU (a one-rank NCCL group): the dispatch puts the
routed rows in expert order and the library's kernel runs on them through
row_to_token, so every (token, slot) row must equal, bit for bit, the row
the direct grouped call computes for the same routing (same kernel, same
per-row arithmetic), and stay within the oracle's tolerance."""
import datetime
import socket

import numpy as np
import pytest
import torch

import oracle as orc
import synth
from parity import assert_rows_close

pytestmark = pytest.mark.gpu

gbw = pytest.importorskip("grouped_bit_weight_b200")
from gpu_util import bits, packed_weights, to_dev  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def one_rank_group():
    import torch.distributed as dist
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("fmt,mode,T", [("nf4", "auto", 1), ("nf4", "gemm", 300),
                                        ("mxfp4", "auto", 300), ("mxfp4", "gemv", 3)])
def test_ep_matches_the_direct_grouped_call(one_rank_group, fmt, mode, T):
    from grouped_bit_weight_b200.ep import ExpertParallel, ep_grouped_gemm
    E, N, K, k = 16, 192, 512, 4
    codes, scale, wdec = packed_weights(fmt, E, N, K, 0.05, 90)
    x_bits = synth.to_bf16_bits(synth.normal((T, K), 91))
    rng = np.random.default_rng(92)
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int64)
    x, w, s = to_dev(x_bits), to_dev(codes), to_dev(scale)
    ep = ExpertParallel(E)
    y = ep_grouped_gemm(ep, x, torch.from_numpy(ids).cuda(), w, s, fmt=fmt, mode=mode)
    torch.cuda.synchronize()
    assert gbw.device_status() == 0
    assert tuple(y.shape) == (T, k, N)
    # the same routing through the direct call
    flat = ids.reshape(-1)
    order = np.argsort(flat, kind="stable")
    off = np.searchsorted(flat[order], np.arange(E + 1)).astype(np.int32)
    r2t = (order // k).astype(np.int32)
    fn = gbw.gnf4_grouped_gemm if fmt == "nf4" else gbw.gmxfp4_grouped_gemm
    direct = bits(fn(x, w, s, to_dev(off), to_dev(r2t), mode=mode))
    got = bits(y).reshape(T * k, N)[order]
    assert np.array_equal(got, direct)
    _, ref = orc.grouped_forward(x_bits, wdec, off, r2t, want_f64=True)
    assert_rows_close(got, ref, what=f"ep {fmt} {mode}")
