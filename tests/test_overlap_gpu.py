"""params.overlap_previous: a call whose attention kernel may start while the
work before it on the stream still runs (programmatic dependent launch), for
callers that process the queries in independent slices ("Krea 2 TileMix
Attention (FP16/INT8 tiles)": the queries go through the core in slices).

The slices write disjoint rows of one output, so overlapping them must change
nothing: the result equals the ordinary calls' bit for bit. And the overlapped
call still completes after the work before it: a copy enqueued right after the
last slice, with no synchronisation in between, sees every slice's rows."""
import pytest
import torch

import diffusion_transformer_attention_bidirectional_b200 as K
from synth import inputs as S

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def sliced(c, q, k, v, g, rows, overlap, **opts):
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device=DEV)
    geo = dict(text_len=c.text_len, grid_h=c.grid_h, grid_w=c.grid_w, mode=c.mode, out=out, **opts)
    for i, s in enumerate(range(0, c.seq_len, rows)):
        K.attention(q, k, v, g, q_start=s, q_len=min(rows, c.seq_len - s), overlap_previous=overlap and i > 0,
                    **geo)
    snapshot = out.clone()  # enqueued right after the last slice, no synchronisation in between
    torch.cuda.synchronize()
    return out, snapshot


@pytest.mark.parametrize("mode", ["dense", "scanline"])
def test_overlapped_slices_equal_ordered_slices(mode):
    c = S.Case("ov", 2, 8, 2, 128, 512, 64, 64, dtype="bf16", mode=mode, seed=401, gate=True, window=11)
    q, k, v, g = (t.to(DEV) for t in S.make_inputs(c))
    opts = {"window": 11} if mode == "scanline" else {}
    ref, _ = sliced(c, q, k, v, g, 1024, False, **opts)
    for _ in range(3):
        out, snap = sliced(c, q, k, v, g, 1024, True, **opts)
        assert torch.equal(out, ref)
        assert torch.equal(snap, ref)


def test_overlap_ignored_where_a_quantiser_runs_first():
    # TileMix: the call's quantiser writes the workspace the attention reads, so the
    # attention keeps ordinary stream order even when the caller allows overlap
    c = S.Case("ov_tm", 1, 8, 2, 128, 256, 32, 32, dtype="f16", mode="tilemix", seed=402,
               qk_dist="normal_koffset", pattern="band", percentage=0.5, smooth_k=True)
    q, k, v, g = (None if t is None else t.to(DEV) for t in S.make_inputs(c))
    ref, _ = sliced(c, q, k, v, g, 384, False, pattern="band", percentage=0.5, smooth_k=True)
    out, snap = sliced(c, q, k, v, g, 384, True, pattern="band", percentage=0.5, smooth_k=True)
    assert torch.equal(out, ref) and torch.equal(snap, ref)
