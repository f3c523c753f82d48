"""The seeded input generators that the oracle and the GPU path share: the
same seed gives the same tensors, the recipe's shapes and statistics hold, and
random tile maps carry exactly the requested number of 2:4 tiles."""
import numpy as np
import torch

from sparse_gemm_wanda_b200 import inputs


def test_same_seed_same_tensors():
    assert torch.equal(inputs.weight(64, 128, 5), inputs.weight(64, 128, 5))
    o = inputs.outlier_channels(256, 5)
    assert torch.equal(inputs.activations(8, 256, 5, o, role=2), inputs.activations(8, 256, 5, o, role=2))
    assert not torch.equal(inputs.activations(8, 256, 5, o, role=1), inputs.activations(8, 256, 5, o, role=2))
    assert not torch.equal(inputs.weight(64, 128, 5), inputs.weight(64, 128, 6))


def test_recipe_statistics():
    w = inputs.weight(512, 512, 1).float()
    assert w.dtype == torch.float32 and abs(w.std().item() - 0.02) < 0.001
    o = inputs.outlier_channels(4096, 1)
    assert o.numel() == 41 and len(set(o.tolist())) == 41  # round(1 % of 4096)
    assert inputs.outlier_channels(256, 1, count=3).numel() == 3
    x = inputs.activations(2048, 4096, 1, o).float()
    mask = torch.zeros(4096, dtype=torch.bool)
    mask[o] = True
    assert abs(x[:, ~mask].std().item() - 1.0) < 0.02
    assert abs(x[:, mask].std().item() - 20.0) < 0.5


def test_chunked_activations_first_block_is_the_plain_draw():
    o = inputs.outlier_channels(256, 3)
    xc = inputs.activations_chunked(40, 256, 3, o, role=4, chunk=16)
    assert xc.shape == (40, 256) and xc.dtype == torch.bfloat16
    assert torch.equal(xc[:16], inputs.activations(16, 256, 3, o, role=4))
    assert torch.equal(xc[16:32], inputs.activations(16, 256, 3, o, role=4 + 100000))
    assert torch.equal(xc[32:], inputs.activations(8, 256, 3, o, role=4 + 200000))


def test_random_map_has_exactly_the_requested_tiles():
    for nt, ns in [(16, 8), (70, 0), (70, 70), (1024, 614), (33, 17)]:
        m = inputs.random_map(nt, ns, 9).numpy().view(np.uint32)
        bits = [(int(m[t // 32]) >> (t % 32)) & 1 for t in range(nt)]
        assert sum(bits) == ns
        assert m.size == (nt + 31) // 32
        # no bits past the last tile
        assert sum(bin(int(v)).count("1") for v in m) == ns


def test_floor_rule_for_tile_counts():
    assert inputs.n_sparse_tiles(0.6, 1024) == 614
    assert inputs.n_sparse_tiles(0.6, 2752) == 1651
    assert inputs.n_sparse_tiles(1.0, 16) == 16 and inputs.n_sparse_tiles(0.0, 16) == 0


def test_workloads_name_the_five_configurations():
    wl = inputs.workloads()
    assert set(wl) == {"tiny", "llama7b-decode", "llama7b-prefill", "llama13b-prefill", "llama7b-block"}
    assert [(m.N, m.K) for m in wl["llama7b-decode"].matrices] == [(4096, 4096), (11008, 4096)]
    assert wl["llama7b-decode"].tokens == [1, 4, 16]
    blk = wl["llama7b-block"]
    assert blk.calib_tokens == 128 * 2048 and blk.fractions == [0.6]
    # q/k/v share one input, gate/up another
    groups = {m.name: m.input_group for m in blk.matrices}
    assert groups["q"] == groups["k"] == groups["v"] != groups["o"]
    assert groups["gate"] == groups["up"] != groups["down"]
