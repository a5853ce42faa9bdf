"""The synthetic MoE routing (host-side input generation): every token gets
top-k distinct experts, rows come sorted by expert, each expert's run is
padded to whole 128-row blocks, and every block's first row is a routed row."""
import torch

import workloads as W


def test_routing_layout():
    T, E, k = 777, 20, 6
    rt, re = W.moe_routing(T, E, k, seed=11, skew=1.5)
    assert rt.numel() == re.numel() and rt.numel() % W.MOE_BLOCK == 0
    real = re >= 0
    assert torch.equal(real, rt >= 0)
    assert int(real.sum()) == T * k
    # each token: k rows, k distinct experts
    pairs = torch.stack([rt[real], re[real].long()], 1)
    assert torch.unique(pairs, dim=0).shape[0] == T * k
    assert torch.equal(torch.bincount(rt[real], minlength=T), torch.full((T,), k))
    # sorted by expert, runs padded to blocks, block heads routed
    ex = re[real].long()
    assert bool((ex[1:] >= ex[:-1]).all())
    heads = re.view(-1, W.MOE_BLOCK)[:, 0]
    assert bool((heads >= 0).all())
    for b in range(heads.numel()):
        blk = re[b * W.MOE_BLOCK:(b + 1) * W.MOE_BLOCK]
        assert bool(((blk == heads[b]) | (blk == -1)).all())
        pad = (blk == -1).nonzero()
        if pad.numel():  # padding only at the end of a block
            assert bool((blk[int(pad[0]):] == -1).all())


def test_routing_is_seeded_and_gather():
    a = W.moe_routing(100, 8, 2, seed=3)
    b = W.moe_routing(100, 8, 2, seed=3)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    x = torch.arange(100 * 4, dtype=torch.float32).view(100, 4).to(torch.bfloat16)
    g = W.gather_rows(x, a[0])
    for r in range(g.shape[0]):
        t = int(a[0][r])
        assert torch.equal(g[r], x[t] if t >= 0 else torch.zeros(4, dtype=torch.bfloat16))
