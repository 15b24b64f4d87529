"""The device conversions of the append kernel against the oracle's codec
(which is itself pinned to ml_dtypes / torch casts): exhaustive over every
float in the ranges where rounding decisions happen, sampled elsewhere."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def _dev_encode(fn, x: np.ndarray) -> np.ndarray:
    import nvfp4_kv_cache_append_b200 as nv
    xd = torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()
    out = torch.empty(xd.numel(), dtype=torch.uint8, device="cuda")
    fn(xd.data_ptr(), out.data_ptr(), xd.numel(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _binade_floats(lo_exp, hi_exp, stride=1):
    lo = np.float32(2.0 ** lo_exp).view(np.uint32)
    hi = np.float32(2.0 ** hi_exp).view(np.uint32)
    return np.arange(lo, hi, stride, dtype=np.uint32).view(np.float32)


@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_e2m1_exhaustive_decision_range(sign):
    import nvfp4_kv_cache_append_b200 as nv
    y = _binade_floats(-3, 4) * np.float32(sign)          # 58.7M floats
    for part in np.array_split(y, 4):
        assert np.array_equal(_dev_encode(nv.nvkv_encode_e2m1, part), oracle.e2m1_encode_array(part))


def test_e2m1_random_bits():
    import nvfp4_kv_cache_append_b200 as nv
    rng = np.random.default_rng(0)
    y = rng.integers(0, 0x7F800000, size=8_000_000, dtype=np.uint32).view(np.float32)
    y = np.concatenate([y, -y, np.float32([0.0, -0.0, 6.0, 3.4e38, 1e-45])])
    assert np.array_equal(_dev_encode(nv.nvkv_encode_e2m1, y), oracle.e2m1_encode_array(y))


def test_block_scale_exhaustive_normal_range():
    import nvfp4_kv_cache_append_b200 as nv
    t = _binade_floats(-12, 9)                            # 176M floats up to 512
    for part in np.array_split(t, 16):
        assert np.array_equal(_dev_encode(nv.nvkv_encode_block_scale, part),
                              oracle.block_scale_code_array(part))


def test_block_scale_tiny_and_huge():
    import nvfp4_kv_cache_append_b200 as nv
    rng = np.random.default_rng(1)
    t = np.concatenate([
        rng.integers(0, np.float32(2.0 ** -12).view(np.uint32), 4_000_000, dtype=np.uint32).view(np.float32),
        rng.integers(np.float32(512.0).view(np.uint32), 0x7F800000, 4_000_000, dtype=np.uint32).view(np.float32),
        np.float32([0.0, 448.0, 464.0, 3.4e38])])
    assert np.array_equal(_dev_encode(nv.nvkv_encode_block_scale, t), oracle.block_scale_code_array(t))
