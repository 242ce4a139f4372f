"""The FFN demo of the cf-1.com post (§6.1) on this package's kernels: gate and up in
full, SwiGLU, the down projection reduced to the 64-neuron blocks of largest mean |h|.

Parity per op on the GPU's own intermediates (the oracle is fed the GPU's bf16 h, so a
near-tie in h cannot flip a block): the full gate/up products, the kept blocks bit for
bit, the reduced down projection within the float bar; keep ratio 1 gives the full FFN.
"""
import numpy as np
import pytest
import torch

import oracle
import rmm_synth
from parity import assert_close

pytestmark = pytest.mark.gpu
H, M, BLOCK = 1024, 4096, 64


@pytest.fixture(scope="module")
def demo():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from input_adaptive_reduced_rmm_b200 import rmm
    from input_adaptive_reduced_rmm_b200.ffn_demo import FfnBlockReduce

    rmm.lib()
    Wg = rmm_synth.weights(M, H, 141, std=0.02)
    Wu = rmm_synth.weights(M, H, 142, std=0.02)
    Wd = rmm_synth.weights(H, M, 143, std=0.02)
    return FfnBlockReduce, (Wg, Wu, Wd)


@pytest.mark.parametrize("T", [1, 4])
@pytest.mark.parametrize("keep", [0.5, 0.25])
def test_ffn_demo_per_op(demo, T, keep):
    cls, (Wg, Wu, Wd) = demo
    f = cls(Wg.cuda(), Wu.cuda(), Wd.cuda(), block=BLOCK, keep=keep, fused_swiglu=False)
    x = rmm_synth.normal((T, H), 144 + T)
    y, blocks, h = f.forward(x.cuda())
    torch.cuda.synchronize()
    b = f._bufs[T]
    # the fused form (SwiGLU applied as gate/up are folded) gives the same h, kept blocks and y
    ff = cls(Wg.cuda(), Wu.cuda(), Wd.cuda(), block=BLOCK, keep=keep)
    y2, blocks2, h2 = ff.forward(x.cuda())
    torch.cuda.synchronize()
    assert torch.equal(h2.view(torch.int16), h.view(torch.int16))
    assert torch.equal(blocks2, blocks) and torch.equal(y2.view(torch.int16), y.view(torch.int16))
    assert_close(b["gate"].cpu(), oracle.linear(x, Wg, 1.0)[0], "gate (full)")
    assert_close(b["up"].cpu(), oracle.linear(x, Wu, 1.0)[0], "up (full)")
    assert_close(h.cpu(), oracle.swiglu(b["gate"].cpu(), b["up"].cpu()), "swiglu")
    yo, bo = oracle.linear_blocks(h.cpu(), Wd, keep, block=BLOCK, block_score="mean")
    assert blocks.cpu().numpy().tolist() == bo.tolist()
    assert_close(y.cpu(), yo, f"down reduced T={T} keep={keep}")


def test_ffn_demo_full_keep_is_the_full_ffn(demo):
    cls, (Wg, Wu, Wd) = demo
    f = cls(Wg.cuda(), Wu.cuda(), Wd.cuda(), block=BLOCK, keep=1.0)
    x = rmm_synth.normal((1, H), 145)
    y, blocks, h = f.forward(x.cuda())
    torch.cuda.synchronize()
    assert blocks.cpu().numpy().tolist() == list(range(M // BLOCK))
    yo, _ = oracle.linear(h.cpu(), Wd, 1.0)
    assert_close(y.cpu(), yo, "keep = 1")
    assert torch.allclose(y.float(), f.forward_dense(x.cuda()).float(), rtol=2e-2, atol=2e-3)
