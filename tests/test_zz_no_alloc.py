"""gptq_quantize_layer_noalloc: the quantize entry point for callers that cannot give the
library device scratch memory (for example code running under a memory pool it does not own,
or code that must not call cudaMalloc because it can synchronise the device). It uses the
library's fixed device array instead of a workspace. This file is collected last on purpose.

The test calls it twice in a row through the C ABI and compares both results with the
workspace entry point (same kernels, same inputs: the results must be identical, which is
tighter than the parity tolerance), checks that the second (warm) call changes neither torch's
allocated bytes nor the device's free memory, and checks the size limit."""
import ctypes

import numpy as np
import pytest
import torch

import datagen

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _outputs(m, n, bits, gs):
    G = n // gs if gs else 1
    return (torch.full((m, n * bits // 32), -1, dtype=torch.int32, device=DEV),
            torch.full((m, G), -1.0, device=DEV),
            torch.full((m, G), 255, dtype=torch.uint8, device=DEV),
            torch.full((m,), -1.0, dtype=torch.float64, device=DEV))


@pytest.mark.parametrize("wl,scale", [("attn", 0.5), ("mlp_down", 0.25)])
def test_noalloc_matches_workspace_entry_twice(wl, scale):
    import post_weight_quantization_06_b200 as g
    L = datagen.WORKLOADS[wl](device=DEV, scale=scale)
    m, n = L.m, L.n
    H = torch.zeros(n, n, device=DEV)
    g.gptq_hessian_accumulate(H, L.X)
    U = torch.empty(n, n, device=DEV)
    lam = torch.empty(1, device=DEV)
    g.gptq_prepare_hinv(H, L.lambda_rel, U, lam, g.workspace(g.GPTQ_OP_PREPARE_HINV, m, n))
    ref = _outputs(m, n, L.bits, L.group_size)
    g.gptq_quantize_layer(L.W, U, L.bits, L.group_size, L.block_size, *ref,
                          g.workspace(g.GPTQ_OP_QUANTIZE, m, n, 0, L.block_size))
    g.gptq_sync_status()
    for call in range(2):
        out = _outputs(m, n, L.bits, L.group_size)
        torch.cuda.synchronize()
        held, free = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
        g.gptq_quantize_layer_noalloc(L.W, U, L.bits, L.group_size, L.block_size, *out)
        g.gptq_sync_status()
        held_after, free_after = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
        if call == 1:
            # the warm call takes no device memory: neither through torch nor from the driver
            assert held_after == held
            assert free_after == free
        for a, b in zip(ref, out):
            assert torch.equal(a, b)


def test_noalloc_rejects_layers_beyond_the_scratch():
    import post_weight_quantization_06_b200 as g
    m, n, B = 4096, 8192, 128      # 128 MiB of working copy > 64 MiB
    assert g.gptq_workspace_size(g.GPTQ_OP_QUANTIZE, m, n, 0, B) > g.NOALLOC_SCRATCH_BYTES
    P = ctypes.c_void_p(256)
    before = g.gptq_launch_count()
    st = g._lib.gptq_quantize_layer_noalloc(P, 1, m, n, P, 4, 128, B, P, P, P, None, None)
    assert st == g.GPTQ_ERR_ARG
    assert g.gptq_launch_count() == before
