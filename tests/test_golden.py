"""The values the pages print (tests/golden/page_constants.json) hold in the oracle."""
import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")


def _load():
    with open(GOLDEN) as f:
        return json.load(f)


def test_every_entry_is_cited():
    g = _load()
    for k, v in g.items():
        if not k.startswith("_"):
            assert "cite" in v and v["cite"], k


def test_shape_rule_cases_in_oracle(orc):
    """ceil(out/128) x ceil(in/128) for each (in, out) of the pages' models; the
    weight is [out, in] as in nn.Linear."""
    g = _load()
    for k_in, n_out, kb, nb in g["shape_rule_cases"]["value"]:
        assert (-(-n_out // 128), -(-k_in // 128)) == (nb, kb)
        # exercise the oracle on a thin slice with the same K (and the full N when small)
        n = n_out if n_out * k_in <= 4 * 1024 * 1024 else 129
        w = np.zeros((n, k_in), dtype=np.uint16)
        for fmt in (0, 1):
            _, ws = orc.quantize_weight(w, fmt)
            assert ws.shape == (-(-n // 128), kb)


def test_group_and_block_width(orc):
    g = _load()
    assert g["weight_block_size"]["value"] == [128, 128]
    assert g["activation_group_width"]["value"] == 128
    x = np.zeros((1, 129), dtype=np.uint16)
    _, xs = orc.quantize_act(x, 0)
    assert xs.shape == (1, 2)  # a group boundary every 128 channels


def test_tested_block_size_in_oracle(orc):
    """The non-default block size the pages' tests cover: 1 x 32 activation
    groups and 32 x 32 weight blocks, scales shaped by the same ceil rule."""
    g = _load()
    bs = g["tested_block_size"]["value"]
    assert bs == [32, 32]
    x = np.zeros((2, 80), dtype=np.uint16)
    w = np.zeros((40, 80), dtype=np.uint16)
    for fmt in (0, 1):
        _, xs = orc.quantize_act(x, fmt, bs[1])
        _, ws = orc.quantize_weight(w, fmt, bs[0])
        assert xs.shape == (2, 3) and ws.shape == (2, 3)


def test_expert_workload_uses_the_blackwell_expert_format():
    import bench
    g = _load()
    assert bench.moe_config(0, 0)["scale_fmt"] == g["blackwell_expert_scale_fmt"]["value"]
