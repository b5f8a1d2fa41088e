"""krea_attn_fwd_noalloc: the attention for callers that cannot allocate device
memory while they run (an arena that forbids cudaMalloc/cudaFree, a host
framework that owns all device memory, a serving loop that must not block on
the allocator). It keeps the tile map and the TileMix workspace in the
library's fixed device array, so its results must equal krea_attn_fwd's, call
after call, and shapes that do not fit must be refused before any launch.

This file is collected last on purpose: it runs after every other test, and it
must also pass alone in a fresh process."""
import ctypes

import pytest
import torch

import diffusion_transformer_attention_bidirectional_b200 as K
from diffusion_transformer_attention_bidirectional_b200 import _lib
from synth import inputs as S

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 64 << 20


def _params(case, q, k, v, g, out, status):
    p = K.make_params(case.batch, case.q_heads, case.kv_heads, case.head_dim, case.text_len, case.grid_h,
                      case.grid_w, in_dtype=case.dtype, out_dtype="f32", pattern=case.pattern,
                      percentage=case.percentage, band_blocks=case.band_blocks, smooth_k=case.smooth_k,
                      window=case.window, tile_aligned=case.tile_aligned, text_pad=case.text_pad,
                      debug_wait_limit=400_000_000)
    for arr, t in ((p.q_stride, q), (p.k_stride, k), (p.v_stride, v), (p.out_stride, out)):
        arr[0], arr[1], arr[2] = t.stride()[:3]
    if g is not None:
        p.gate_stride[0], p.gate_stride[1], p.gate_stride[2] = g.stride()[:3]
    p.status = status.data_ptr()
    return p


def noalloc(case, q, k, v, g):
    out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    status = torch.zeros(1, dtype=torch.int32, device=q.device)
    p = _params(case, q, k, v, g, out, status)
    rc = _lib.lib().krea_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                          g.data_ptr() if g is not None else None, out.data_ptr(),
                                          case.text_len, case.grid_h, case.grid_w, _lib.MODE[case.mode],
                                          ctypes.byref(p), torch.cuda.current_stream().cuda_stream)
    return rc, out, status


def reference_call(case, q, k, v, g):
    return K.attention(q, k, v, g, text_len=case.text_len, grid_h=case.grid_h, grid_w=case.grid_w,
                       mode=case.mode, pattern=case.pattern, percentage=case.percentage,
                       band_blocks=case.band_blocks, smooth_k=case.smooth_k, window=case.window,
                       tile_aligned=case.tile_aligned, text_pad=case.text_pad)


CASES = [
    S.Case("na_tilemix", 1, 8, 2, 128, 200, 30, 30, dtype="f16", mode="tilemix", seed=41,
           qk_dist="normal_koffset", pattern="band", percentage=0.5, band_blocks=1),
    S.Case("na_scanline", 1, 4, 2, 128, 100, 20, 20, dtype="bf16", mode="scanline", seed=42, window=5,
           gate=True),
    S.Case("na_tilemix_again", 1, 8, 2, 128, 300, 25, 33, dtype="bf16", mode="tilemix", seed=43,
           qk_dist="normal_koffset", pattern="one", band_blocks=2),
    S.Case("na_dense", 1, 4, 1, 64, 16, 8, 8, dtype="f16", mode="dense", seed=45, gate=True),
]


def test_noalloc_matches_fwd_call_after_call():
    # The same kernels on the same inputs, with the tile map built into the array by
    # the device builder (bit-identical to the cached host map) and the TileMix
    # workspace in the array: the outputs equal krea_attn_fwd's bit for bit, on two
    # calls in a row of every case (consecutive calls share the array; each must
    # stand on its own). params.workspace stays NULL throughout, TileMix included.
    dev = torch.device("cuda:0")
    for case in CASES:
        q, k, v, g = (t.to(dev) if t is not None else None for t in S.make_inputs(case))
        ref = reference_call(case, q, k, v, g)
        for _ in range(2):
            rc, out, status = noalloc(case, q, k, v, g)
            torch.cuda.synchronize()
            assert rc == 0, K._lib.lib().krea_attn_error_string(rc)
            assert int(status.item()) == 0
            assert torch.equal(out, ref), f"{case.name}: max |diff| {float((out - ref).abs().max())}"


def test_noalloc_allocates_nothing():
    # Once the kernels are loaded (a first call of each kind), further calls leave
    # both torch's allocator and the device's free memory exactly where they were.
    dev = torch.device("cuda:0")
    inputs = []
    for case in CASES:
        q, k, v, g = (t.to(dev) if t is not None else None for t in S.make_inputs(case))
        out = torch.empty(q.shape, dtype=torch.float32, device=dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        p = _params(case, q, k, v, g, out, status)
        assert not p.workspace  # no caller workspace, TileMix included
        inputs.append((case, q, k, v, g, out, status, p))

    def run_all():
        for case, q, k, v, g, out, status, p in inputs:
            rc = _lib.lib().krea_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                  g.data_ptr() if g is not None else None, out.data_ptr(),
                                                  case.text_len, case.grid_h, case.grid_w, _lib.MODE[case.mode],
                                                  ctypes.byref(p), torch.cuda.current_stream().cuda_stream)
            assert rc == 0, K._lib.lib().krea_attn_error_string(rc)

    run_all()
    torch.cuda.synchronize()
    torch_before = torch.cuda.memory_allocated(dev)
    free_before, _ = torch.cuda.mem_get_info(dev)
    for _ in range(3):
        run_all()
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated(dev) == torch_before
    assert torch.cuda.mem_get_info(dev)[0] == free_before
    assert all(int(x[6].item()) == 0 for x in inputs)


def test_noalloc_refuses_shapes_beyond_its_array():
    # 48/12-head TileMix over 512 + 96x96 tokens needs ~105 MB of workspace
    case = S.Case("na_big", 1, 48, 12, 128, 512, 96, 96, dtype="f16", mode="tilemix", seed=44,
                  pattern="band")
    p = K.make_params(1, 48, 12, 128, 512, 96, 96, in_dtype="f16")
    assert K.workspace_bytes("tilemix", 512, 96, 96, p) > SCRATCH_BYTES
    dev = torch.device("cuda:0")
    L = case.seq_len
    q = torch.zeros(1, L, 48, 128, dtype=torch.float16, device=dev)
    k = torch.zeros(1, L, 12, 128, dtype=torch.float16, device=dev)
    rc, _, status = noalloc(case, q, k, k, None)
    torch.cuda.synchronize()
    assert rc == _lib.ERR_TOO_LARGE
    assert int(status.item()) == 0


def test_noalloc_writes_the_same_lse():
    case = CASES[1]  # scanline, gated
    dev = torch.device("cuda:0")
    q, k, v, g = (t.to(dev) if t is not None else None for t in S.make_inputs(case))
    want = torch.full((1, case.q_heads, case.seq_len), float("nan"), dtype=torch.float32, device=dev)
    K.attention(q, k, v, g, text_len=case.text_len, grid_h=case.grid_h, grid_w=case.grid_w, mode=case.mode,
                window=case.window, tile_aligned=case.tile_aligned, text_pad=case.text_pad, lse=want)
    got = torch.full_like(want, float("nan"))
    out = torch.empty(q.shape, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    p = _params(case, q, k, v, g, out, status)
    p.lse = got.data_ptr()
    rc = _lib.lib().krea_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), g.data_ptr(), out.data_ptr(),
                                          case.text_len, case.grid_h, case.grid_w, _lib.MODE[case.mode],
                                          ctypes.byref(p), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == 0 and int(status.item()) == 0
    assert torch.equal(got, want)  # the same kernel on the same inputs: bit for bit
