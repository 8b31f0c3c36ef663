"""Host threads calling the library at the same time, each on its own CUDA
stream (ctypes releases the interpreter lock for the duration of a call).
The threads make the calls first, so when this file runs alone their first
launches race on the per-device set-up and the kernels' shared-memory
opt-in.  Every thread's results must equal, bit
for bit, what the same calls give one after another, and the device error
word must stay clear."""
import threading

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

gbw = pytest.importorskip("grouped_bit_weight_b200")
from gpu_util import bits, packed_weights, to_dev  # noqa: E402


def _case(fmt, E, N, K, T, k, mode, seed):
    codes, scale, _ = packed_weights(fmt, E, N, K, 0.05, seed)
    rng = np.random.default_rng(seed + 1)
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).reshape(-1)
    order = np.argsort(ids, kind="stable")
    off = np.searchsorted(ids[order], np.arange(E + 1)).astype(np.int32)
    r2t = (order // k).astype(np.int32)
    x = synth.to_bf16_bits(synth.normal((T, K), seed + 2))
    fn = gbw.gnf4_grouped_gemm if fmt == "nf4" else gbw.gmxfp4_grouped_gemm
    args = [to_dev(a) for a in (x, codes, scale, off, r2t)]
    return lambda: fn(*args, mode=mode)


def test_concurrent_host_threads_match_serial_calls():
    # distinct kernels per thread: GEMV shapes, tensor-core shapes, formats
    cases = [_case("nf4", 16, 256, 512, 2, 2, "gemv", 10),
             _case("mxfp4", 16, 256, 576, 300, 4, "gemm", 20),
             _case("nf4", 8, 192, 1024, 200, 2, "gemm", 30),
             _case("mxfp4", 8, 128, 320, 3, 2, "auto", 40)]
    got = [[None] * 3 for _ in cases]
    errors = []
    barrier = threading.Barrier(len(cases))

    def worker(i):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                barrier.wait()
                outs = [cases[i]() for _ in range(3)]
            s.synchronize()
            got[i] = [bits(o) for o in outs]
        except Exception as exc:  # reported below
            errors.append(exc)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(len(cases))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(120)
    assert not errors, errors
    assert gbw.device_status() == 0
    # the same calls one after another, on the default stream
    serial = [bits(c()) for c in cases]
    torch.cuda.synchronize()
    for i, ref in enumerate(serial):
        for rep in got[i]:
            assert np.array_equal(rep, ref), f"case {i}"
