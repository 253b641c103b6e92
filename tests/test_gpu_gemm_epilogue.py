"""The tf32x3 GEMM's two epilogues round alike: slices written through the C tensor map (a bulk
store for beta = 0, an fp32 add-reduction in L2 for beta = 1) give bit-identical layer
outputs to the read-modify-write epilogue (GPTQ_GEMM_RMW_EPILOGUE, read once per process, so
that run is a child process)."""
import os
import subprocess
import sys

import pytest
import torch

import datagen

pytestmark = pytest.mark.gpu
DEV = "cuda"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_CHILD = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
import datagen
import post_weight_quantization_06_b200 as g
L = datagen.attn(device="cuda", scale=0.5)
H = torch.load(sys.argv[2]).cuda()
out = g.quantize_layer(L.W, H=H, bits=L.bits, group_size=L.group_size, block_size=128)
torch.save({k: out[k].cpu() for k in ("U", "codes", "scales", "zeros", "loss")}, sys.argv[3])
"""


def test_tensor_map_epilogue_is_bit_identical_to_read_modify_write(tmp_path):
    import post_weight_quantization_06_b200 as g
    L = datagen.attn(device=DEV, scale=0.5)
    ref = g.quantize_layer(L.W, L.X, bits=L.bits, group_size=L.group_size, block_size=128)
    h_path, o_path = str(tmp_path / "H.pt"), str(tmp_path / "out.pt")
    torch.save(ref["H"].cpu(), h_path)
    # the same layer from the same H in this process (tensor-map epilogue by default) ...
    out = g.quantize_layer(L.W, H=ref["H"].clone(), bits=L.bits, group_size=L.group_size,
                           block_size=128)
    # ... and in a child process with the read-modify-write epilogue everywhere
    env = dict(os.environ, GPTQ_GEMM_RMW_EPILOGUE="1")
    subprocess.run([sys.executable, "-c", _CHILD, ROOT, h_path, o_path], env=env, check=True,
                   timeout=600)
    rmw = torch.load(o_path)
    for key in ("U", "codes", "scales", "zeros", "loss"):
        assert torch.equal(out[key].cpu(), rmw[key]), key
