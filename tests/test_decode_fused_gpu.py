"""GPU parity of the one-kernel decode step (mla_attn_decode_fused: attention, split merge and output
projection in one grid with a grid-wide hand-off): bit for bit against mla_attn_decode_out, whose
kernels compute the same arithmetic in the same order, and against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from deepseek_mla_latent_b200 import workloads as wl

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from deepseek_mla_latent_b200 import mla
    from gpu_util import assert_close, to_dev


def _both(w, num_splits=0, calls=2):
    d = mla.dims_from(w.dims)
    dev = to_dev(w)
    q_abs = mla.absorb_q(d, dev["q"], dev["wkv_b"])
    ref = mla.attn_decode_out(d, q_abs, dev["q"], dev["kv"], dev["pe"], dev["cu_k"], dev["max_k"], dev["wkv_b"],
                              num_splits=num_splits)
    ws = mla.decode_fused_workspace(d, w.batch, dev["max_k"], num_splits)
    outs = []
    for _ in range(calls):
        out = torch.full_like(ref, float("nan"))
        mla.attn_decode_fused(d, q_abs, dev["q"], dev["kv"], dev["pe"], dev["cu_k"], dev["max_k"], dev["wkv_b"],
                              out=out, ws=ws, num_splits=num_splits)
        mla.device_status()
        outs.append(out)
    # the control words are back at zero after every call
    assert torch.count_nonzero(ws[:256]).item() == 0
    return ref, outs


@pytest.mark.parametrize("seqlens,splits", [([1000, 260], 7), ([4096, 33], 0), ([0, 70, 0], 3), ([1, 200, 777], 2)])
def test_fused_equals_two_kernel_path_bit_for_bit(seqlens, splits):
    w = wl.make_workload("fz", wl.V3, [1] * len(seqlens), seqlens, seed=61)
    ref, outs = _both(w, splits)
    for o in outs:
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16))
    assert_close(outs[-1].float().cpu().numpy().astype(np.float64), oracle.workload_naive(w), "bf16", "out")


def test_fused_single_split_and_too_many_units_take_the_two_kernel_path():
    """One split (no merge) and a plan with more CTAs than SMs run mla_attn_decode_out's kernels
    on the same workspace; results still match it bit for bit."""
    w = wl.make_workload("fz1", wl.V3, [1, 1], [300, 50], seed=62)
    ref, outs = _both(w, 1)
    assert torch.equal(outs[0].view(torch.int16), ref.view(torch.int16))
    w = wl.make_workload("fz2", wl.V3, [1] * 40, [700] * 40, seed=63)
    ref, outs = _both(w, 4)
    assert torch.equal(outs[0].view(torch.int16), ref.view(torch.int16))


def test_full_fused_decode_sampled():
    """The DeepSeek-V3 decode workload (batch 8 x 4096, automatic splits: 144 CTAs) and the
    long-context workload (batch 2 x 131072, 37 splits: 148 CTAs, every SM), checked bit for bit
    against the two-kernel path and against the oracle on one head of every sequence and heads 0,
    63, 64, 127 of one."""
    for idx, row in ((1, 4), (3, 1)):
        w = wl.workload(idx)
        ref, outs = _both(w, 0, calls=2)
        for o in outs:
            assert torch.equal(o.view(torch.int16), ref.view(torch.int16))
        got = outs[-1].float().cpu().numpy().astype(np.float64)
        rng = np.random.default_rng(64 + idx)
        pairs = sorted({(b, int(rng.integers(0, 128))) for b in range(w.batch)} | {(row, h) for h in (0, 63, 64, 127)})
        for (b, h), r in oracle.workload_naive(w, pairs=pairs).items():
            assert_close(got[b:b + 1, h, :], r, "bf16", f"workload {idx} seq {b} head {h}")
