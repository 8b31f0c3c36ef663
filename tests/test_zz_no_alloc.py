"""The fused NF4 expert pass for callers that cannot hand the library device
memory at call time (an engine plugin whose device memory the engine already
owns, a serving loop that forbids allocation after warm-up):
gnf4_grouped_expert_mlp_noalloc keeps h in the library's own fixed scratch
array instead of a caller workspace.

Called through the C ABI with raw pointers, it must give what
gnf4_grouped_expert_mlp gives with a caller workspace, within the tolerance
the matmul tests use, on two calls in a row: a decode-sized call (bandwidth
GEMV path) and then a larger one (tensor-core path), so the second call also
shows that nothing left in the shared scratch by the first one leaks in.
This file is collected last on purpose."""
import ctypes as C

import pytest
import torch

import synth
from parity import assert_rows_close, bf16_bits_to_f64

gbw = pytest.importorskip("grouped_bit_weight_b200")
from gpu_util import bits, packed_weights, to_dev  # noqa: E402

SHAPE = 2  # GBW_ERR_SHAPE


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _noalloc(x, gu, dn, off, r2t, P, H, I, E):
    out = torch.empty((P, H), dtype=torch.bfloat16, device=x.device)
    st = gbw.lib.gnf4_grouped_expert_mlp_noalloc(
        _ptr(x), x.shape[0], H, _ptr(gu[0]), _ptr(gu[1]), _ptr(dn[0]), _ptr(dn[1]), E, I,
        _ptr(off), _ptr(r2t), P, _ptr(out), gbw.MODE_AUTO,
        C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, gbw.lib.gbw_status_string(st).decode()
    return out


@pytest.mark.gpu
def test_no_alloc_entry_matches_the_workspace_entry_on_two_calls():
    E, H, I = 8, 2048, 768
    gu = [to_dev(a) for a in packed_weights("nf4", E, 2 * I, H, 0.02, 81)[:2]]
    dn = [to_dev(a) for a in packed_weights("nf4", E, H, I, 0.02, 82)[:2]]
    calls = [(synth.decode_routing(E, 8, 0), 1, 84),            # P = 8: GEMV path
             (synth.uniform_routing(64, E, 2, seed=83), 64, 85)]  # P = 128: tensor cores
    for (off, r2t), T, seed in calls:
        x = to_dev(synth.to_bf16_bits(synth.normal((T, H), seed)))
        d_off, d_r2t = to_dev(off), to_dev(r2t)
        P = int(off[-1])
        ref, _ = gbw.gnf4_grouped_expert_mlp(x, gu[0], gu[1], dn[0], dn[1], d_off, d_r2t)
        got = _noalloc(x, gu, dn, d_off, d_r2t, P, H, I, E)
        torch.cuda.synchronize()
        assert gbw.device_status() == 0
        assert_rows_close(bits(got), bf16_bits_to_f64(bits(ref)),
                          what=f"no-allocation entry, P={P}")


def test_no_alloc_entry_rejects_problems_larger_than_its_scratch():
    """P * I above the scratch's 2,097,152 values is refused before anything
    reaches the GPU (runs without one)."""
    p = C.c_void_p(16)
    st = gbw.lib.gnf4_grouped_expert_mlp_noalloc(p, 4096, 2048, p, p, p, p, 8, 768, p, None,
                                                 4096, p, 0, None)
    assert st == SHAPE
    assert b"scratch" in gbw.lib.gbw_status_string(st)
