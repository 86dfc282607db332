"""Parity of whole MoE layers at the benchmark's sizes, in the benchmark's
call shapes, on a subset of layers spread over each sweep (the first, a
middle and the last layer).

* Qwen3-30B-A3B refit (MXFP8, swizzled, 16 experts per call, layers 0, 23,
  47): the first gate_up and the first down call of the layer compared with
  the oracle completely, and one expert of every other call.
* Qwen3-235B-A22B prequantization (128 experts per call, layers 0, 46, 93),
  the six calls of a layer -- MXFP8, NVFP4 with the per-tensor amax computed
  and NVFP4 with that amax given, for gate_up and down: one whole call per
  layer compared with the oracle (layer 0 gate_up MXFP8, layer 46 down NVFP4
  computed, layer 93 gate_up NVFP4 given), three experts of every other call,
  and every expert's amax against torch's maximum of the same tensor.

Layers are drawn by ``synth.moe_layer`` from their own seeds, exactly as the
benchmark regenerates them.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import assert_bytes_equal, host_bits, oracle_threads

pytestmark = pytest.mark.gpu

qz = pytest.importorskip("nvfp4_quantization_moe_b200")
SWZ = qz.SF_SWIZZLED


def oracle_check(xs_dev, got, fmt, mode=None, amax_in=None, what=""):
    """Compare (q, sf[, amax]) of each expert with the oracle on the host copy."""
    hosts = [host_bits(x) for x in xs_dev]
    ofmt = oracle.MXFP8 if fmt == qz.FMT_MXFP8 else oracle.NVFP4
    ref = oracle.quantize_grouped(hosts, ofmt, SWZ, mode if mode is not None else oracle.NVFP4_PER_ROW, amax_in,
                                  threads=oracle_threads())
    for i, (g, r) in enumerate(zip(got, ref)):
        assert_bytes_equal(g[0].reshape(-1), r[0].reshape(-1), f"{what} expert {i} payload")
        assert_bytes_equal(g[1], r[1], f"{what} expert {i} scales")
        if fmt == qz.FMT_NVFP4 and mode == qz.NVFP4_PER_TENSOR_COMPUTE:
            assert np.array_equal(g[2].view(np.uint32), r[2].view(np.uint32)), f"{what} expert {i} amax"


@pytest.mark.parametrize("layer", [0, 23, 47])
def test_qwen3_30b_refit_layers(layer):
    cfg = synth.QWEN3_30B
    E, per_call = cfg["experts"], 16
    for proj in ("gate_up", "down"):
        stack = synth.moe_layer(cfg, layer, proj)
        rows, cols = cfg[proj]
        nsf = qz.sf_bytes(rows, cols, qz.FMT_MXFP8, SWZ)
        q = torch.empty((E, rows, cols), dtype=torch.uint8, device="cuda")
        sf = torch.empty((E, nsf), dtype=torch.uint8, device="cuda")
        for s in range(0, E, per_call):
            tab = qz.ExpertTable([qz.Entry(stack[e], q[e], sf[e]) for e in range(s, s + per_call)])
            qz.quantize_grouped_mxfp8(tab, SWZ)
        torch.cuda.synchronize()
        full = list(range(per_call)) if layer == 0 else []
        sample = sorted(set(full + [s + (layer + 5 * s // per_call) % per_call for s in range(0, E, per_call)]))
        got = [(q[e].cpu().numpy(), sf[e].cpu().numpy()) for e in sample]
        oracle_check([stack[e] for e in sample], got, qz.FMT_MXFP8, what=f"30B layer {layer} {proj}")
        del stack, q, sf
        torch.cuda.empty_cache()


LAYER_FULL = {0: ("gate_up", "mxfp8"), 46: ("down", "nvfp4_compute"), 93: ("gate_up", "nvfp4_given")}


@pytest.mark.parametrize("layer", [0, 46, 93])
def test_qwen3_235b_prequant_layers(layer):
    cfg = synth.QWEN3_235B
    E = cfg["experts"]
    for proj in ("gate_up", "down"):
        stack = synth.moe_layer(cfg, layer, proj)
        rows, cols = cfg[proj]
        xs = list(stack.unbind(0))
        mx = qz.alloc_outputs(xs, qz.FMT_MXFP8, SWZ)
        nv = qz.alloc_outputs(xs, qz.FMT_NVFP4, SWZ, qz.NVFP4_PER_TENSOR_COMPUTE)
        nv_tab = qz.ExpertTable(nv)
        qz.quantize_grouped_mxfp8(qz.ExpertTable(mx), SWZ)
        qz.quantize_grouped_nvfp4(nv_tab, qz.NVFP4_PER_TENSOR_COMPUTE, SWZ)
        torch.cuda.synchronize()
        amax = torch.cat([e.amax for e in nv])
        assert torch.equal(amax, stack.float().abs().amax(dim=(1, 2))), f"235B layer {layer} {proj} amax"
        nmx = qz.sf_bytes(rows, cols, qz.FMT_MXFP8, SWZ)
        nnv = qz.sf_bytes(rows, cols, qz.FMT_NVFP4, SWZ)
        full_proj, full_mode = LAYER_FULL[layer]
        sample = [(layer * 7) % E, 64, E - 1 - layer % 5]
        pick = lambda mode: list(range(E)) if (proj, mode) == (full_proj, full_mode) else sample  # noqa: E731
        sel = pick("mxfp8")
        oracle_check([xs[i] for i in sel], [(mx[i].q.cpu().numpy(), mx[i].sf[:nmx].cpu().numpy()) for i in sel],
                     qz.FMT_MXFP8, what=f"235B layer {layer} {proj} MXFP8")
        sel = pick("nvfp4_compute")
        oracle_check([xs[i] for i in sel],
                     [(nv[i].q.cpu().numpy(), nv[i].sf[:nnv].cpu().numpy(), nv[i].amax.cpu().numpy()) for i in sel],
                     qz.FMT_NVFP4, qz.NVFP4_PER_TENSOR_COMPUTE, what=f"235B layer {layer} {proj} NVFP4 computed")
        # requantization with the amax just computed (the benchmark's third call)
        for e in nv:
            e.q.fill_(0x5A)
            e.sf.fill_(0x5A)
        qz.quantize_grouped_nvfp4(nv_tab, qz.NVFP4_PER_TENSOR_GIVEN, SWZ)
        torch.cuda.synchronize()
        sel = pick("nvfp4_given")
        oracle_check([xs[i] for i in sel], [(nv[i].q.cpu().numpy(), nv[i].sf[:nnv].cpu().numpy()) for i in sel],
                     qz.FMT_NVFP4, qz.NVFP4_PER_TENSOR_GIVEN, [float(nv[i].amax[0]) for i in sel],
                     what=f"235B layer {layer} {proj} NVFP4 given")
        del stack, xs, mx, nv, nv_tab, amax
        torch.cuda.empty_cache()
