"""GPU conversion: the kernels' fp32 -> fp16/bf16 step against the oracle
over ALL 2^32 float32 bit patterns, and on arrays with special values."""

import numpy as np
import pytest
import torch

import paged_kv_cache_321_b200 as K

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kv_dtype", ["f16", "bf16"])
def test_exhaustive_bit_patterns(orc, kv_dtype):
    chunk = 1 << 28
    out = torch.empty(chunk, dtype=torch.int16, device="cuda")
    host = torch.empty(chunk, dtype=torch.int16, pin_memory=True)
    for start in range(0, 1 << 32, chunk):
        K.convert_bits(start, chunk, kv_dtype, out)
        host.copy_(out)
        got = host.numpy().view(np.uint16)
        want = orc.convert_range(start, chunk, kv_dtype)
        if not np.array_equal(got, want):
            i = int(np.argmax(got != want))
            raise AssertionError(f"{kv_dtype}: pattern {start + i:#010x}: gpu {got[i]:#06x} oracle {want[i]:#06x}")


@pytest.mark.parametrize("kv_dtype", ["f16", "bf16"])
def test_array_with_special_values(orc, kv_dtype):
    rng = np.random.default_rng(17)
    x = rng.standard_normal(100001).astype(np.float32) * np.float32(1e3)
    special = np.array([0x7FC00000, 0x7F800001, 0xFFFFFFFF, 0x7F800000, 0xFF800000, 0x00000001, 0x80000000,
                        0x477FF000, 0x33000000, 0x387FC000, 0x7F7FFFFF], dtype=np.uint32).view(np.float32)
    x[:len(special)] = special
    xt = torch.from_numpy(x).cuda()
    out = torch.empty(x.size, dtype=torch.int16, device="cuda")
    K.convert_f32(xt, out, kv_dtype)
    assert np.array_equal(out.cpu().numpy().view(np.uint16), orc.convert(x, kv_dtype))
