"""Stream ordering of the overlapped data-parallel gradient exchange
(GradExchanger) on one GPU, with a stand-in collective in place of NCCL:
the exchange must read a layer's gradients only after the kernels that
wrote them, and the caller's stream must see the exchanged values after
finish().  The stand-in records what it read and adds the other rank's
(identical) contribution, after a delay that makes a missing wait show."""
import pytest
import torch

from transformer_layer_pre_b200.dp import FlatGrads, GradExchanger

pytestmark = pytest.mark.gpu

DELAY_CYCLES = 200_000_000   # ~0.1 s at 2 GHz


def test_exchange_waits_for_the_layer_and_the_caller_waits_for_the_exchange():
    dev = torch.device("cuda", 0)
    seen = []

    def standin_allreduce(t):
        torch.cuda._sleep(DELAY_CYCLES)      # a slow collective
        seen.append(t.clone())               # what the collective read
        t.add_(t)                            # the other rank holds the same values

    layers = [FlatGrads(64, 256, dev) for _ in range(3)]
    main = torch.cuda.current_stream(dev)
    ex = GradExchanger(allreduce=standin_allreduce, world=2)
    for l in reversed(range(3)):
        torch.cuda._sleep(DELAY_CYCLES // 4)  # a slow "backward" of layer l
        layers[l].flat.fill_(float(l + 1))
        ex.submit(layers[l], main)
    ex.finish(main)
    after = [g.flat.clone() for g in layers]  # read on the caller's stream
    torch.cuda.synchronize()
    assert len(seen) == 3
    for k, l in enumerate(reversed(range(3))):
        assert torch.all(seen[k] == float(l + 1)), "the exchange read the gradients before they were written"
    for l in range(3):
        assert torch.all(after[l] == float(l + 1)), "the caller read the gradients before the exchange ended"
