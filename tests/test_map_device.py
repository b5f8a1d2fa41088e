"""The device map builder (three kernels on the stream) against the oracle's
brute-force per-pair enumeration, bit for bit, on the host tests' geometries;
and its refusal to write past the caller's arrays."""
import ctypes

import numpy as np
import pytest
import torch

import diffusion_transformer_attention_bidirectional_b200 as K
from diffusion_transformer_attention_bidirectional_b200 import _lib
from oracle import krea_oracle as ko
from synth.inputs import Case

from test_map import SCANLINE_GEOMS

pytestmark = pytest.mark.gpu


def device_map(mode, T, H, W, **opts):
    rp, col, kind = K.get_map_device(mode, T, H, W, **opts)
    torch.cuda.synchronize()
    rp = rp.cpu().numpy()
    nnz = int(rp[-1])
    return rp, col[:nnz].cpu().numpy(), kind[:nnz].cpu().numpy()


def oracle_map(mode, T, H, W, **opts):
    return ko.tile_map(Case("m", 1, 1, 1, 128, T, H, W, mode=mode, **opts)).csr()


def assert_same(a, b, what):
    for x, y, name in zip(a, b, ("row_ptr", "col", "kind")):
        assert np.array_equal(np.asarray(x), np.asarray(y)), f"{what}: {name}"


def test_scanline_device_map():
    rng = np.random.default_rng(11)
    geoms = [dict(T=T, H=H, W=W, window=w, tile_aligned=ta, text_pad=pad) for T, H, W, w, ta, pad in SCANLINE_GEOMS]
    for _ in range(40):
        T = int(rng.integers(0, 900))
        geoms.append(dict(T=T, H=int(rng.integers(1, 40)), W=int(rng.integers(1, 70)),
                          window=int(rng.integers(0, 20)) * 2 + 1, tile_aligned=bool(rng.integers(0, 2)),
                          text_pad=0 if rng.integers(0, 2) else int(np.ceil(max(T, 1) / 128) * 128)))
    for g in geoms:
        o = dict(window=g["window"], tile_aligned=g["tile_aligned"], text_pad=g["text_pad"])
        assert_same(device_map("scanline", g["T"], g["H"], g["W"], **o),
                    oracle_map("scanline", g["T"], g["H"], g["W"], **o), str(g))


def test_tilemix_and_dense_device_map():
    for pattern, pct, band in [("band", 0.5, 2), ("band", 0.75, 2), ("band", 0.0, 2), ("band", 1.0, 2),
                               ("one", 0.5, 2), ("zero", 0.5, 2), ("band", 0.3, 0), ("band", 0.61, 5)]:
        for T, H, W in [(512, 64, 64), (300, 20, 30), (77, 16, 16), (0, 32, 32)]:
            o = dict(pattern=pattern, percentage=pct, band_blocks=band)
            assert_same(device_map("tilemix", T, H, W, **o), oracle_map("tilemix", T, H, W, **o),
                        f"tilemix {pattern} {pct} {band} {T} {H} {W}")
    for T, H, W in [(16, 8, 8), (512, 64, 64), (300, 60, 60), (0, 1, 1), (1000, 0, 0)]:
        assert_same(device_map("dense", T, H, W), oracle_map("dense", T, H, W), f"dense {T} {H} {W}")


def test_device_map_full_size_configs():
    # 4 MP band (132 tiles a side): equal to the host builder, 7938 INT8 tiles
    o = dict(pattern="band", percentage=0.5, band_blocks=2)
    d = device_map("tilemix", 512, 128, 128, **o)
    assert_same(d, K.get_map("tilemix", 512, 128, 128, **o), "4 MP band vs host")
    assert int((d[2] & _lib.KIND_INT8).astype(bool).sum()) == 7938
    o = dict(window=11, tile_aligned=True, text_pad=512)
    assert_same(device_map("scanline", 512, 128, 128, **o), oracle_map("scanline", 512, 128, 128, **o), "4 MP scan")


def test_device_map_respects_capacity():
    params = K.make_params(1, 1, 1, 128, 300, 60, 60, window=11)
    nt, nnz = K.map_size("scanline", 300, 60, 60, params)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    params.status = status.data_ptr()
    row_ptr = torch.zeros(nt + 1, dtype=torch.int32, device="cuda")
    col = torch.full((nnz,), -7, dtype=torch.int32, device="cuda")
    kind = torch.full((nnz,), 9, dtype=torch.uint8, device="cuda")
    rc = _lib.lib().krea_attn_build_map_device(300, 60, 60, _lib.MODE["scanline"], ctypes.byref(params),
                                               row_ptr.data_ptr(), col.data_ptr(), kind.data_ptr(), nnz - 1,
                                               torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == 0
    assert int(status.item()) == _lib.ERR_DEVICE_BOUNDS
    assert int(row_ptr[-1].item()) == nnz  # row_ptr is written either way
    assert bool((col == -7).all()) and bool((kind == 9).all())  # nothing past the caller's capacity
