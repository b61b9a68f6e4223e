"""Host-side launch-shape choice (no GPU): the split-KV chunk count of the attention."""
from long_context_sparse_indexer_b200 import launch


def test_one_split_when_the_layers_fill_the_gpu():
    # 32 tokens x 2 CTAs x 2 concurrent layers = 128 CTAs: one wave without splitting
    assert launch.split_for(32, 128, 2564, layers=2) == 1
    assert launch.split_for(256, 128, 2564, layers=2) == 1
    assert launch.split_for(2048, 128, 2564) == 1


def test_few_tokens_split_to_fill_the_gpu():
    n = launch.split_for(4, 128, 3076)
    assert n > 1
    assert 2 * 4 * n <= launch.B200_SMS          # still one wave
    assert 3076 / n >= 64                         # chunks stay at least two tiles long


def test_concurrent_layers_count_against_the_wave():
    # 16 tokens: one layer alone fills the GPU with 9 splits (144 CTAs); two layers at once
    # would need two waves, so fewer splits win
    assert launch.split_for(16, 128, 2564, layers=1) == 9
    assert launch.split_for(16, 128, 2564, layers=2) < 9
    assert launch.split_for(16, 128, 2564, layers=3) == launch.split_for(16, 128, 2564, layers=2)


def test_split_bounds():
    for T in (1, 3, 7, 33, 1000):
        for cap in (64, 388, 2564, 8192):
            n = launch.split_for(T, 128, cap)
            assert 1 <= n <= 32
            assert n == 1 or cap / n >= 64
    assert launch.split_for(5, 64, 2564) >= 1                  # warp-MMA kernel shapes
