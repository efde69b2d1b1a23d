"""batq_linear_grouped: independent linears in one quantiser launch and one CTA-pair GEMM launch.

* Every activation takes the quantiser kernel its own batq_linear call would take (the tensor-core
  ones share one launch, the CUDA-core ones run as side-by-side launches), and the GEMMs of one tile
  configuration share one launch: the grouped call must give the same workspace codes and scales
  and the same outputs as batq_linear, bit for bit, for every shape.
* Small shapes are also checked against the oracle (codes within the parity bound, outputs within
  1e-4 * sum |a||w| of the fp64 GEMM of those codes).
* Groups whose GEMMs do not share a configuration (mixed S classes, mixed output types) run them
  one after another and must still equal batq_linear bit for bit.
"""

import numpy as np
import pytest
import torch

from mxfp4_w4a4_post_block_b200 import batq as BQ
from mxfp4_w4a4_post_block_b200 import workloads as WL
from oracle import batq_oracle as O
import gpu_util as GU
import parity as PT

pytestmark = pytest.mark.gpu


def _linear(i, S, N, M, x_dtype="bf16", out_dtype=torch.float32):
    w = WL.custom(S, N, M, 500 + i, x_dtype=x_dtype, with_w=False)
    g = torch.Generator(device="cuda").manual_seed(600 + i)
    B, ratios = GU.params(w)
    wc, wsc = BQ.empty_act_buffers(M, N)
    wc.random_(0, 256, generator=g)
    wsc.random_(116, 136, generator=g)
    out = torch.full((S, M), float("nan"), dtype=out_dtype, device="cuda")
    return dict(w=w, X=GU.x_tensor(w), A=w.A, B=B, ratios=ratios, w_codes=wc, w_scales=wsc, M=M, out=out)


def _workspace_parts(ws, linears):
    """Each linear's (codes, MMA scales) views inside the grouped workspace."""
    parts, off = [], 0
    for l in linears:
        S, N = l["w"].S, l["w"].N
        one = BQ.batq_linear_workspace_size(S, N)
        cb = -(-S * (N // 2) // 256) * 256
        parts.append((ws[off:off + S * (N // 2)].view(S, N // 2), ws[off + cb:off + one]))
        off += -(-one // 256) * 256
    return parts


def _run_grouped(linears):
    ws = torch.full((BQ.batq_linear_grouped_workspace_size([(l["w"].S, l["w"].N) for l in linears]),), 0xAB,
                    dtype=torch.uint8, device="cuda")
    BQ.batq_linear_grouped(linears, ws)
    torch.cuda.synchronize()
    assert BQ.batq_device_error() == 0
    return ws


def _run_single(l):
    ws = torch.full((BQ.batq_linear_workspace_size(l["w"].S, l["w"].N),), 0xCD, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(l["out"])
    BQ.batq_linear(l["X"], l["A"], l["B"], l["ratios"], l["w_codes"], l["w_scales"], l["M"], ws, out)
    torch.cuda.synchronize()
    assert BQ.batq_device_error() == 0
    return ws, out


def _assert_linear_equal(i, l, codes, scales):
    """One linear's grouped codes, scales and output against batq_linear's."""
    ws1, out1 = _run_single(l)
    S, N = l["w"].S, l["w"].N
    assert torch.equal(codes, ws1[:S * (N // 2)].view(S, N // 2)), f"linear {i}: codes"
    cb = -(-S * (N // 2) // 256) * 256
    assert torch.equal(scales, ws1[cb:cb + scales.numel()]), f"linear {i}: scales (padding included)"
    assert torch.equal(l["out"], out1), f"linear {i}: output"


def _assert_equal_to_batq_linear(linears, ws):
    for i, (l, (codes, scales)) in enumerate(zip(linears, _workspace_parts(ws, linears))):
        _assert_linear_equal(i, l, codes, scales)


def _assert_oracle_parity(label, l, codes, scales):
    w = l["w"]
    c_h = codes.cpu().numpy()
    a_sc = O.scales_from_mma_layout(scales.cpu().numpy(), w.S, w.k)
    act = O.quant_act(w.x, w.A, w.B, w.alpha_min, w.alpha_max)
    PT.assert_quant_parity(c_h, a_sc, act, label, cond=PT.condition_scale(w.x, w.A, w.B))
    ref, T = O.gemm(c_h, a_sc, l["w_codes"].cpu().numpy(),
                    O.scales_from_mma_layout(l["w_scales"].cpu().numpy(), w.M, w.k))
    PT.assert_gemm_parity(l["out"].float().cpu().numpy(), ref, T, label)


def test_tensor_core_shapes_equal_batq_linear_bit_for_bit():
    # every one of these has >= 6 x 148 tensor-core tiles, so batq_linear uses the same transform;
    # K of 4096 and 12288, M ragged (1040), S ragged (3500), one output tile column (M = 256)
    shapes = [(4096, 4096, 1024), (1280, 12288, 512), (3500, 4096, 1040), (4096, 4096, 256)]
    linears = [_linear(i, *shp) for i, shp in enumerate(shapes)]
    ws = _run_grouped(linears)
    _assert_equal_to_batq_linear(linears, ws)


def test_bf16_output_group_equals_batq_linear():
    shapes = [(4096, 4096, 512), (1536, 12288, 384)]
    linears = [_linear(10 + i, *shp, out_dtype=torch.bfloat16) for i, shp in enumerate(shapes)]
    ws = _run_grouped(linears)
    _assert_equal_to_batq_linear(linears, ws)


def test_small_shapes_match_batq_linear_and_the_oracle():
    # below six tensor-core tiles per SM: the CUDA-core transform, one launch each, side by side
    shapes = [(200, 512, 272), (129, 1024, 256), (300, 768, 1024), (640, 4096, 512), (257, 64, 16)]
    linears = [_linear(20 + i, *shp) for i, shp in enumerate(shapes)]
    ws = _run_grouped(linears)
    for i, (l, (codes, scales)) in enumerate(zip(linears, _workspace_parts(ws, linears))):
        _assert_oracle_parity(f"group linear {i}", l, codes, scales)
    _assert_equal_to_batq_linear(linears, ws)


def test_mixed_quantiser_kernels_in_one_group():
    # two activations for the tensor-core kernel (one grouped launch) and three for the CUDA-core one
    shapes = [(4096, 4096, 512), (200, 512, 272), (1280, 12288, 256), (640, 4096, 512), (300, 768, 1024)]
    linears = [_linear(60 + i, *shp) for i, shp in enumerate(shapes)]
    ws = _run_grouped(linears)
    _assert_equal_to_batq_linear(linears, ws)


@pytest.mark.parametrize("case", ["fp32_input", "short_S", "mixed_out"])
def test_groups_that_do_not_qualify_run_the_linears_own_kernels(case):
    if case == "fp32_input":
        linears = [_linear(30, 300, 1024, 512, x_dtype="f32"), _linear(31, 2048, 4096, 256)]
    elif case == "short_S":
        linears = [_linear(32, 4096, 4096, 512), _linear(33, 16, 4096, 1024), _linear(34, 128, 512, 256)]
    else:
        linears = [_linear(35, 4096, 4096, 512), _linear(36, 4096, 4096, 256, out_dtype=torch.bfloat16)]
    ws = _run_grouped(linears)
    _assert_equal_to_batq_linear(linears, ws)


def test_full_group_of_eight_and_repeat():
    shapes = [(4096, 4096, 512), (4096, 4096, 256), (1280, 12288, 256), (4096, 4096, 128),
              (4096, 4096, 1024), (3584, 4096, 256), (4096, 4096, 384), (1280, 12288, 512)]
    linears = [_linear(40 + i, *shp) for i, shp in enumerate(shapes)]
    ws = _run_grouped(linears)
    first = [l["out"].clone() for l in linears]
    for l in linears:
        l["out"].fill_(float("nan"))
    _run_grouped(linears)
    for i, (a, l) in enumerate(zip(first, linears)):
        assert torch.equal(a, l["out"]), f"linear {i}: not reproducible"
    _assert_equal_to_batq_linear(linears, ws)


@pytest.mark.parametrize("layout", [BQ.BATQ_SCALES_MMA, BQ.BATQ_SCALES_LINEAR])
def test_grouped_quantiser_equals_batq_quant_act(layout):
    """Tensor-core-sized activations (one grouped launch) and small ones (side-by-side CUDA-core
    launches) write what the single calls write."""
    shapes = [(4096, 4096), (1280, 12288), (3500, 4096), (200, 512), (16, 4096)]
    acts, refs = [], []
    for i, (S, N) in enumerate(shapes):
        l = _linear(70 + i, S, N, 128)
        c, s = BQ.empty_act_buffers(S, N, layout)
        c.fill_(0xAB)
        s.fill_(0xAB)
        acts.append(dict(X=l["X"], A=l["A"], B=l["B"], ratios=l["ratios"], codes=c, scales=s))
        c1, s1 = BQ.empty_act_buffers(S, N, layout)
        s1.fill_(0xCD)
        BQ.batq_quant_act(l["X"], l["A"], l["B"], l["ratios"], c1, s1, layout)
        refs.append((c1, s1))
    BQ.batq_quant_act_grouped(acts, layout)
    torch.cuda.synchronize()
    assert BQ.batq_device_error() == 0
    for i, (a, (c1, s1)) in enumerate(zip(acts, refs)):
        assert torch.equal(a["codes"], c1), f"activation {i}: codes"
        assert torch.equal(a["scales"], s1), f"activation {i}: scales"


@pytest.mark.parametrize("case", ["pair", "with_short_S"])
def test_grouped_gemm_equals_batq_gemm_mxfp4(case):
    g = torch.Generator(device="cuda").manual_seed(80)
    shapes = [(4096, 1024, 4096), (300, 272, 12288), (2048, 4096, 512)]
    if case == "with_short_S":
        shapes.append((16, 2048, 4096))
    gemms, refs = [], []
    for S, M, N in shapes:
        a, sa = BQ.empty_act_buffers(S, N)
        a.random_(0, 256, generator=g)
        sa.random_(116, 136, generator=g)
        w, sw = BQ.empty_act_buffers(M, N)
        w.random_(0, 256, generator=g)
        sw.random_(116, 136, generator=g)
        out = torch.full((S, M), float("nan"), dtype=torch.float32, device="cuda")
        gemms.append(dict(a_codes=a, a_scales=sa, w_codes=w, w_scales=sw, S=S, M=M, N=N, out=out))
        ref = torch.empty_like(out)
        BQ.batq_gemm_mxfp4(a, sa, w, sw, S, M, N, ref)
        refs.append(ref)
    BQ.batq_gemm_mxfp4_grouped(gemms)
    torch.cuda.synchronize()
    assert BQ.batq_device_error() == 0
    for i, (gm, ref) in enumerate(zip(gemms, refs)):
        assert torch.equal(gm["out"], ref), f"product {i} {shapes[i]}"


def _pair_launch_splits(tiles):
    """The pair GEMM's rule: a last round of whole tiles that fills at most half of the clusters runs
    as 256 x 128 half tiles."""
    clusters = torch.cuda.get_device_properties(0).multi_processor_count // 2
    rem = tiles % clusters
    return 0 < rem and 2 * rem <= clusters


def test_half_tile_last_round_equals_whole_tiles():
    """down_proj alone (16 x 16 = 256 pair tiles, 34 in the last round on 74 clusters) runs its last
    round as half tiles; grouped with a 20-tile companion (276 tiles, 54 in the last round) the same
    tiles run whole.  Each output element is one K accumulation either way: the bits must agree, for
    the companion (split when alone) too."""
    g = torch.Generator(device="cuda").manual_seed(81)
    shapes = [(4096, 4096, 12288), (1024, 1280, 4096)]
    tiles = [-(-S // 256) * -(-M // 256) for S, M, _ in shapes]
    assert _pair_launch_splits(tiles[0]) and _pair_launch_splits(tiles[1])
    assert not _pair_launch_splits(sum(tiles))
    gemms, refs = [], []
    for S, M, N in shapes:
        a, sa = BQ.empty_act_buffers(S, N)
        a.random_(0, 256, generator=g)
        sa.random_(116, 136, generator=g)
        w, sw = BQ.empty_act_buffers(M, N)
        w.random_(0, 256, generator=g)
        sw.random_(116, 136, generator=g)
        out = torch.full((S, M), float("nan"), dtype=torch.float32, device="cuda")
        gemms.append(dict(a_codes=a, a_scales=sa, w_codes=w, w_scales=sw, S=S, M=M, N=N, out=out))
        ref = torch.full_like(out, float("nan"))
        BQ.batq_gemm_mxfp4(a, sa, w, sw, S, M, N, ref)
        refs.append(ref)
    BQ.batq_gemm_mxfp4_grouped(gemms)
    torch.cuda.synchronize()
    assert BQ.batq_device_error() == 0
    for i, (gm, ref) in enumerate(zip(gemms, refs)):
        assert not torch.isnan(ref).any(), f"product {i}: output not fully written"
        assert torch.equal(gm["out"], ref), f"product {i} {shapes[i]}"


def test_layer_workload_as_the_bench_runs_it():
    """The seven S = 8192 linears of the layer workload (q, k, v, o, gate, up, down) through one grouped
    call, as the bench times them: every output, code and scale equals batq_linear's bit for bit (each
    of these shapes takes the tensor-core transform in batq_linear too), and rows of the down linear
    match the oracle."""
    linears = []
    for j in range(len(WL.LAYER_LINEARS)):
        w = WL.layer_linear(j, with_w=False)
        g = torch.Generator(device="cuda").manual_seed(900 + j)
        B, ratios = GU.params(w)
        wc, wsc = BQ.empty_act_buffers(w.M, w.N)
        wc.random_(0, 256, generator=g)
        wsc.random_(118, 134, generator=g)
        out = torch.full((w.S, w.M), float("nan"), dtype=torch.float32, device="cuda")
        linears.append(dict(w=w, X=GU.x_tensor(w), A=w.A, B=B, ratios=ratios, w_codes=wc, w_scales=wsc, M=w.M,
                            out=out))
    ws = _run_grouped(linears)
    parts = _workspace_parts(ws, linears)
    for i, (l, (codes, scales)) in enumerate(zip(linears, parts)):
        _assert_linear_equal(i, l, codes, scales)
    # sampled rows of the down linear (K = 12288) against the oracle's fp64 GEMM of the grouped codes
    l, (codes, scales) = linears[-1], parts[-1]
    w = l["w"]
    rows = np.sort(np.random.default_rng(901).choice(w.S, 48, replace=False))
    c_h = codes.cpu().numpy()
    a_sc = O.scales_from_mma_layout(scales.cpu().numpy(), w.S, w.k)
    ref, T = O.gemm_rows(c_h, a_sc, l["w_codes"].cpu().numpy(),
                         O.scales_from_mma_layout(l["w_scales"].cpu().numpy(), w.M, w.k), rows)
    PT.assert_gemm_parity(l["out"].cpu().numpy()[rows], ref, T, "layer down, grouped")


@pytest.mark.parametrize("shapes", [
    [(16, 4096, 4096), (16, 1024, 4096), (9, 12288, 4096), (1, 272, 512)],  # S <= 16 (decode, BN = 16)
    [(32, 1024, 4096), (17, 512, 1024)],                                     # S <= 32
    [(40, 2048, 4096), (64, 256, 320)],                                      # S <= 64, ragged K stage
    [(100, 1024, 4096), (128, 256, 512), (65, 512, 1024)],                   # S <= 128 (BN = 256)
])
def test_small_S_gemm_group_equals_single_calls(shapes):
    """Products of one small-S tile configuration share one launch of the single-CTA kernel."""
    g = torch.Generator(device="cuda").manual_seed(sum(s[0] for s in shapes))
    gemms, refs = [], []
    for S, M, N in shapes:
        a, sa = BQ.empty_act_buffers(S, N)
        a.random_(0, 256, generator=g)
        sa.random_(116, 136, generator=g)
        w, sw = BQ.empty_act_buffers(M, N)
        w.random_(0, 256, generator=g)
        sw.random_(116, 136, generator=g)
        out = torch.full((S, M), float("nan"), dtype=torch.float32, device="cuda")
        gemms.append(dict(a_codes=a, a_scales=sa, w_codes=w, w_scales=sw, S=S, M=M, N=N, out=out))
        ref = torch.empty_like(out)
        BQ.batq_gemm_mxfp4(a, sa, w, sw, S, M, N, ref)
        refs.append(ref)
    BQ.batq_gemm_mxfp4_grouped(gemms)
    torch.cuda.synchronize()
    assert BQ.batq_device_error() == 0
    for i, (gm, ref) in enumerate(zip(gemms, refs)):
        assert torch.equal(gm["out"], ref), f"product {i} {shapes[i]}"


def test_decode_layer_group():
    """A decode step of the layer's seven linears at S = 16 through one grouped call (side-by-side
    CUDA-core quantiser launches, one single-CTA GEMM launch): equal to batq_linear bit for bit, and
    within the oracle's bounds."""
    linears = []
    for j, (name, N, M) in enumerate(WL.LAYER_LINEARS):
        linears.append(_linear(950 + j, 16, N, M))
    ws = _run_grouped(linears)
    for i, (l, (codes, scales)) in enumerate(zip(linears, _workspace_parts(ws, linears))):
        _assert_oracle_parity(f"decode group {i}", l, codes, scales)
    _assert_equal_to_batq_linear(linears, ws)
    # repeated back to back: the side-by-side launches of one call must not overtake the previous call
    for _ in range(3):
        BQ.batq_linear_grouped(linears, ws)
    torch.cuda.synchronize()
    assert BQ.batq_device_error() == 0
    _assert_equal_to_batq_linear(linears, ws)
