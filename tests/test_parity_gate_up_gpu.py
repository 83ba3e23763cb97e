"""GPU parity of the fused gate|up module with the SiLU epilogue ("LLM quantization speed-up", "fused
modules"): awq_pack_gate_up bit-exact against the oracle's pack of the interleaved matrix, and
w4a16_gate_up_silu (GEMV and GEMM modes) against the oracle's fp64 silu(x' Wg^T) * (x' Wu^T).  The shapes
reach every way the decode kernel finishes a row block: one CTA per row block with its warps combining in
shared memory (NI = 1024), whole row blocks per CTA (NI = 14336), and row blocks split between CTAs and
combined in the workspace (NI = 2432: 152 row blocks)."""
import numpy as np
import pytest
import torch

from helpers import assert_epilogue_within_tolerance, sample_pairs
from oracle import oracle as O
import synth
import weight_only_int4_05_b200 as W4

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.float16)


def host_u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def host_u32(t):
    return t.detach().cpu().contiguous().numpy().view(np.uint32)


class GateUpCase:
    def __init__(self, seed, M, NI, K, g=128):
        dg = synth.linear_inputs(seed, 7, 0, 4, M, NI, K)
        du = synth.linear_inputs(seed, 7, 0, 5, M, NI, K)
        self.M, self.NI, self.K, self.g = M, NI, K, g
        self.Wg = dg["W"].view(np.uint16)
        self.Wu = du["W"].view(np.uint16)
        self.xcal = dg["xcal"].view(np.uint16)
        self.x = dg["x"].view(np.uint16)
        self.s = O.act_scale(self.xcal)
        self.xp = O.inv_scale(self.x, self.s)
        self.qg = O.quantize(self.Wg, self.s, g)
        self.qu = O.quantize(self.Wu, self.s, g)

    def packed(self):
        return O.awq_pack(O.interleave_gate_up(self.Wg, self.Wu), self.s, self.g)

    def ab_pairs(self, ms, js):
        """The oracle's fp64 gate and up outputs a, b at the listed pairs (h_ref = silu(a) b)."""
        return (O.linear_pairs_f64(self.xp, *self.qg, ms, js, self.g),
                O.linear_pairs_f64(self.xp, *self.qu, ms, js, self.g))

    def ab_all(self):
        mm, jj = np.meshgrid(np.arange(self.M), np.arange(self.NI), indexing="ij")
        a, b = self.ab_pairs(mm.ravel(), jj.ravel())
        return a.reshape(self.M, self.NI), b.reshape(self.M, self.NI)

    def cuda(self):
        s = W4.awq_act_scale(dev(self.xcal))
        xp = W4.awq_apply_inv_scale(dev(self.x), s)
        pw = W4.awq_pack_gate_up(dev(self.Wg), dev(self.Wu), s, g=self.g)
        return xp, pw


@pytest.mark.parametrize("M,NI,K,g", [(1, 1024, 512, 128), (5, 256, 1024, 128), (16, 2432, 512, 128),
                                      (32, 1024, 256, 64), (1, 2432, 1024, 256), (64, 256, 512, 128),
                                      (200, 1024, 512, 64), (3, 16, 128, 128)])
def test_gate_up_silu_every_output(M, NI, K, g):
    case = GateUpCase(1, M, NI, K, g)
    xp, pw = case.cuda()
    h = W4.w4a16_gate_up_silu(xp, pw)
    torch.cuda.synchronize()
    qw, sc, qz = case.packed()
    assert np.array_equal(host_u32(pw.qweight), qw)
    assert np.array_equal(host_u16(pw.scales), sc)
    assert np.array_equal(host_u32(pw.qzeros), qz)
    assert h.shape == (M, NI)
    a, b = case.ab_all()
    assert_epilogue_within_tolerance(h.float().cpu().numpy(), a, b, f"M={M} NI={NI} K={K} g={g}")
    # the oracle's fused definition agrees with silu(a) b at every output
    assert np.array_equal(O.gate_up_silu_pairs_f64(case.xp, *case.qg, *case.qu, [0], [0], g), O.silu(a[:1, :1].ravel()) * b[:1, :1].ravel())
    assert W4.awq_last_device_status() == 0


def test_gate_up_silu_llama_decode_and_prefill_sampled():
    """Llama-3-8B MLP front half, 4096 -> 2 x 14336: M = 1 (decode, GEMV) and M = 2048 (prefill, GEMM),
    sampled outputs covering the corners and random positions."""
    for M in (1, 2048):
        case = GateUpCase(2, M, 14336, 4096)
        xp, pw = case.cuda()
        h = W4.w4a16_gate_up_silu(xp, pw)
        torch.cuda.synchronize()
        ms, js = sample_pairs(M, 14336, 3000, seed=M)
        a, b = case.ab_pairs(ms, js)
        assert_epilogue_within_tolerance(h.float().cpu().numpy()[ms, js], a, b, f"M={M}")
    assert W4.awq_last_device_status() == 0


def test_gate_up_silu_matches_unfused_composition_in_a_graph():
    """Captured in a CUDA graph with the other calls of the MLP's front half (no host sync): the fused call
    agrees with silu(gate) * up formed from two plain linears on the same packed rows within fp16 rounding
    of the unfused path (which rounds gate and up to fp16 before the product)."""
    case = GateUpCase(3, 1, 4096, 1024)
    xp, pw = case.cuda()
    pg = W4.awq_pack(dev(case.Wg), W4.awq_act_scale(dev(case.xcal)))
    pu = W4.awq_pack(dev(case.Wu), W4.awq_act_scale(dev(case.xcal)))
    h = torch.empty((1, 4096), dtype=torch.float16, device="cuda")
    yg = torch.empty_like(h)
    yu = torch.empty_like(h)
    W4.w4a16_gate_up_silu(xp, pw, out=h)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        W4.w4a16_gate_up_silu(xp, pw, out=h)
        W4.w4a16_linear(xp, pg, out=yg)
        W4.w4a16_linear(xp, pu, out=yu)
    h.zero_()
    graph.replay()
    torch.cuda.synchronize()
    ref = (torch.nn.functional.silu(yg.float()) * yu.float()).cpu().numpy()
    got = h.float().cpu().numpy()
    a, b = case.ab_all()
    bound = 2.0 ** -9 * np.abs(ref) + 2e-3 * (np.abs(yu.float().cpu().numpy()) + np.abs(ref))
    assert np.all(np.abs(got - ref) <= bound)  # the unfused path differs by its two extra fp16 roundings
    assert_epilogue_within_tolerance(got, a, b, "graph")
    del graph


def test_gate_up_argument_checks():
    case = GateUpCase(4, 1, 32, 128)
    xp, pw = case.cuda()
    with pytest.raises(W4.AwqError):
        W4.awq_pack_gate_up(dev(case.Wg[:24]), dev(case.Wu[:24]))  # NI % 16 != 0
    with pytest.raises(ValueError):
        W4.w4a16_gate_up_silu(xp, pw, out=torch.empty((1, 64), dtype=torch.float16, device="cuda"))
