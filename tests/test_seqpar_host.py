"""Host-side checks of the sequence <-> head exchange binding (no GPU): the
destination table and the argument checks that run before any library call."""
import pytest
import torch

from diffusion_transformer_attention_bidirectional_b200 import _lib, seqpar


def test_destinations_table():
    d = seqpar.Destinations([0x1000, 0x2000, 0x3000], (4096 * 12 * 128, 12 * 128, 128, 1), torch.bfloat16)
    assert d.world == 3 and d.strides == (4096 * 12 * 128, 12 * 128, 128)
    ex = d.struct(rank=2, tokens_per_rank=1536)
    assert (ex.world, ex.rank, ex.tokens_per_rank, ex.reserved) == (3, 2, 1536, 0)
    assert [ex.dst[j] for j in range(3)] == [0x1000, 0x2000, 0x3000]
    assert all(ex.dst[j] is None for j in range(3, _lib.EXCHANGE_MAX_RANKS))
    assert list(ex.dst_stride) == [4096 * 12 * 128, 12 * 128, 128]
    with pytest.raises(ValueError):
        seqpar.Destinations([], (1, 1, 1), torch.float16)
    with pytest.raises(ValueError):
        seqpar.Destinations(list(range(1, 18)), (1, 1, 1), torch.float16)


def test_destinations_of_checks_tensors():
    with pytest.raises(ValueError):  # host tensors are not destinations
        seqpar.Destinations.of([torch.zeros(1, 8, 2, 64, dtype=torch.float16)])


def test_sources_are_checked_before_the_library():
    d = seqpar.Destinations([0x1000, 0x2000], (8 * 2 * 64, 2 * 64, 64), torch.float16)
    x = torch.zeros(1, 4, 4, 64, dtype=torch.float16)
    with pytest.raises(ValueError):  # a host tensor
        seqpar.seq_to_heads(x, d, 0)
    with pytest.raises(ValueError):
        seqpar.heads_to_seq(x, d, 0)


def test_ranges_partition():
    for W in (1, 2, 3, 4, 6, 12):
        heads = [h for j in range(W) for h in range(*seqpar.head_range(48, W, j))]
        assert heads == list(range(48))
    toks = [t for r in range(4) for t in range(*seqpar.token_range(1152, r))]
    assert toks == list(range(4608))
