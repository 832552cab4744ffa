"""Host logic of the block-sequential driver: calibration batches of the same
sequence shape are joined (up to a token budget) for one forward, and the
outputs are split back into the caller's batches."""
import torch

from post_weight_quantization_05_b200.driver import BlockSequential


def test_merge_groups_and_round_trip():
    b = BlockSequential(max_tokens=20)
    g = torch.Generator().manual_seed(0)
    xs = [torch.randn(s, generator=g) for s in [(2, 4, 3), (1, 4, 3), (3, 5, 3), (2, 5, 3), (1, 4, 3)]]
    merged, groups = b._merge(xs)
    # same shape joins up to 20 tokens; a shape change or the budget starts a new batch
    assert [tuple(t.shape) for t in merged] == [(3, 4, 3), (3, 5, 3), (2, 5, 3), (1, 4, 3)]
    assert groups == [[2, 1], [3], [2], [1]]
    back = [p for x, gs in zip(merged, groups) for p in x.split(gs)]
    assert len(back) == len(xs) and all(torch.equal(a, c) for a, c in zip(xs, back))


def test_merge_single_batch_is_untouched():
    x = torch.randn(4, 8, 16)
    merged, groups = BlockSequential()._merge([x])
    assert merged[0] is x and groups == [[4]]
