"""GEMM launch timing (GPTQ_FLAG_KERNEL_TIMES) on the GPU: the record fills, clears on read,
counts the column sweep's lazy updates exactly, and leaves every result bit-identical."""
import pytest
import torch

import datagen

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def g():
    import post_weight_quantization_06_b200 as lib
    return lib


def test_kernel_times_count_the_pass_and_change_nothing(g):
    L = datagen.attn(device=DEV, scale=0.5)
    m, n = L.W.shape
    B = 128
    ref = g.quantize_layer(L.W, L.X, bits=L.bits, group_size=L.group_size, block_size=B)
    g.kernel_times()
    g.gptq_set_flags(g.GPTQ_FLAG_KERNEL_TIMES)
    try:
        out = g.quantize_layer(L.W, H=ref["H"].clone(), bits=L.bits, group_size=L.group_size,
                               block_size=B)
    finally:
        g.gptq_set_flags(0)
    kt = g.kernel_times()
    for key in ("U", "codes", "scales", "zeros", "loss", "lam"):
        assert torch.equal(out[key], ref[key]), key
    print({f"{s}/{p}": (v["launches"], round(v["ms"], 3), v["flops"]) for (s, p), v in kt.items()})
    assert ("factor", "tc") in kt and ("sweep", "tc") in kt
    assert all(v["launches"] > 0 and v["ms"] > 0 and v["flops"] > 0 and v["bytes"] > 0
               for v in kt.values())
    # every pair of columns in different panels meets in one multiply-add per row
    sweep = sum(v["flops"] for (s, _), v in kt.items() if s == "sweep")
    assert sweep == m * (n * n - n * B)
    assert g.kernel_times() == {}
    # with the flag clear nothing is noted
    g.quantize_layer(L.W, H=ref["H"].clone(), bits=L.bits, group_size=L.group_size, block_size=B)
    assert g.kernel_times() == {}
