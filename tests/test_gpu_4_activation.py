"""Activation NVFP4 quantizer (nvfp4_quantize_activation) on the GPU vs the CPU
oracle, bit for bit: packed E2M1 codes and E4M3 scales in both the plain and
the swizzled layout of the block-scaled GEMM ("Move NVFP4 GEMM management into
NvFp4LinearKernel", flashinfer.py: scaled_fp4_quant(x, input_global_scale_inv,
is_sf_swizzled_layout=True) and swizzle_blockscale), padding bytes included."""
import numpy as np
import pytest
import torch

import nvfp4_quantized_paged_append_b200 as nk
import oracle
from nvfp4_quantized_paged_append_b200 import workloads as wl
from paged_helpers import u16

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(rows, cols, seed, outliers=False, stride=None):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    width = cols if stride is None else stride
    x = torch.randn((rows, width), generator=g, device=DEV, dtype=torch.float32)
    if outliers:
        ch = torch.randperm(cols, generator=g, device=DEV)[: max(1, cols // 50)]
        x[:, ch] *= 20.0
    x = x.to(torch.bfloat16)[:, :cols]
    amax = float(x.float().abs().amax())
    inv = float(np.float32(448.0 * 6.0) / np.float32(amax))
    return x, inv


@pytest.mark.parametrize("rows,cols,swz,outl,stride", [
    (200, 96, True, False, None),      # padding in both directions
    (200, 96, False, False, None),
    (1, 16, True, False, None),        # one group
    (257, 4096, True, True, None),     # outlier channels, ragged row band
    (130, 512, True, False, 640),      # row stride above cols
    (2048, 4096, True, True, None),    # a slice of the benchmark's shape
])
def test_activation_quantizer_bit_exact(rows, cols, swz, outl, stride):
    x, inv = _inputs(rows, cols, rows + cols, outl, stride)
    n = nk.activation_sf_bytes(rows, cols, swz)
    sf_dev = torch.full((n,), 0xAB, dtype=torch.uint8, device=DEV)     # padding must become 0
    fp4, sf = nk.quantize_activation(x, torch.tensor([inv], device=DEV), swizzled=swz,
                                     out_sf=sf_dev)
    torch.cuda.synchronize()
    ref_fp4, ref_sf = oracle.quantize_activation(np.ascontiguousarray(u16(x)), inv, swizzled=swz)
    assert np.array_equal(fp4.cpu().numpy(), ref_fp4)
    assert np.array_equal(sf.cpu().numpy().reshape(ref_sf.shape), ref_sf)


def test_activation_quantizer_zero_and_tiny_groups():
    """All-zero groups (scale 0, codes 0), a subnormal effective scale and
    values that round to -0 (code 0x8), bit for bit."""
    cols = 64
    x = torch.zeros((4, cols), dtype=torch.float32)
    x[1, :16] = torch.linspace(-1e-30, 1e-30, 16)
    x[2, 16:32] = torch.tensor([6.0, -0.2] + [0.01] * 14)
    x[3] = torch.linspace(-3, 3, cols)
    x = x.to(torch.bfloat16).to(DEV)
    inv = float(np.float32(1.0))
    fp4, sf = nk.quantize_activation(x, torch.tensor([inv], device=DEV), swizzled=False)
    torch.cuda.synchronize()
    ref_fp4, ref_sf = oracle.quantize_activation(np.ascontiguousarray(u16(x)), inv, swizzled=False)
    assert np.array_equal(fp4.cpu().numpy(), ref_fp4)
    assert np.array_equal(sf.cpu().numpy(), ref_sf)
    assert (ref_fp4[0] == 0).all() and (ref_sf[0] == 0).all()
