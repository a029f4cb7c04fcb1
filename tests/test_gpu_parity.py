"""GPU parity of the fused kernels against the CPU oracle, element by
element, on shapes that span several tiles and ragged tails, for every
epilog, both 16-bit types and every tile width the planner can choose."""
import numpy as np
import pytest
import torch

import oracle
from gemm_epilogues_tcgen05_b200 import binding, synth

from _parity import (check_backward, check_forward, check_wgrad, odt, run_backward, run_ffn_step, run_forward,
                     run_wgrad)

pytestmark = pytest.mark.gpu

DT = {"fp16": torch.float16, "bf16": torch.bfloat16}
SHAPES = [(1, 8, 8), (5, 40, 24), (130, 72, 136), (200, 264, 200), (257, 520, 328), (384, 512, 512),
          (300, 640, 136)]  # the last two: ceil(N/32) % 4 == 0, so mask words go out by TMA store
# few-row shapes whose feature tiles are split over several CTAs (stream-K
# segments), with ragged K and N, and one where every CTA owns whole tiles
SKINNY_SHAPES = [(16, 1032, 2048), (100, 264, 1000), (256, 4104, 520), (40, 2056, 64), (1, 11008, 4096)]
FWD_EPILOGS = ["BIAS", "RELU_BIAS", "RELU_AUX_BIAS", "GELU_BIAS", "GELU_AUX_BIAS"]
# CTA-pair shapes: T not a multiple of 256 (the peer CTA's rows partly or
# wholly past T), N not a multiple of 256 (the peer's columns past N)
PAIR_SHAPES = [(300, 264, 136), (600, 520, 328), (1000, 1032, 264), (257, 8, 64), (600, 1024, 328),
               # more than one wave of pair tiles (74 pairs): the last round's tiles are split
               # into column halves; ragged T and N, one with mask words by TMA store
               (1000, 5000, 72), (1024, 5120, 64)]
# kernel variants: the tile kernel at each width, the few-row kernel and the
# CTA-pair tile kernel
VARIANTS = ["tile64", "tile128", "tile192", "tile256", "skinny", "pair"]


def _force(monkeypatch, variant):
    if variant in ("skinny", "pair"):
        monkeypatch.setenv("GEMM_EPI_FORCE_KERNEL", variant)
        monkeypatch.delenv("GEMM_EPI_FORCE_BN", raising=False)
    else:
        monkeypatch.setenv("GEMM_EPI_FORCE_KERNEL", "tile")
        monkeypatch.setenv("GEMM_EPI_FORCE_BN", variant[4:])


def _expect_variant(info, variant, T):
    if (variant == "skinny" and T <= 256) or (variant == "pair" and T <= 128):
        assert info["kernel"] == 1
    elif variant == "pair":
        assert info["kernel"] == 2
    else:
        assert info["kernel"] == 0
        if variant != "skinny":
            assert info["tile_n"] == int(variant[4:])


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("T,N,K", SHAPES)
def test_forward_all_epilogs(monkeypatch, T, N, K, dtype, variant):
    _force(monkeypatch, variant)
    inp = synth.make_shape_inputs(T, N, K, dtype, seed=T * 7 + N + K)
    for ep in FWD_EPILOGS:
        gpu = run_forward(inp, ep, DT[dtype])
        _expect_variant(gpu["info"], variant, T)
        check_forward(inp, ep, DT[dtype], gpu)


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("T,N,K", SHAPES)
def test_backward_drelu_bgrad(monkeypatch, T, N, K, dtype, variant):
    _force(monkeypatch, variant)
    D2 = max(8, (K // 2) // 8 * 8)
    inp = synth.make_shape_inputs(T, N, K, dtype, seed=T * 5 + N + K, D2=D2)
    fwd = run_forward(inp, "RELU_AUX_BIAS", DT[dtype])
    gpu = run_backward(inp, fwd["aux"], DT[dtype])
    _expect_variant(gpu["info"], variant, T)
    check_backward(inp, fwd["aux"], DT[dtype], gpu)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("T,N,K", PAIR_SHAPES)
def test_pair_kernel_ragged(monkeypatch, T, N, K, dtype):
    """CTA-pair kernel on ragged shapes, every epilog, and DRELU_BGRAD twice."""
    _force(monkeypatch, "pair")
    D2 = max(8, (K // 2) // 8 * 8)
    inp = synth.make_shape_inputs(T, N, K, dtype, seed=T + 3 * N + K, D2=D2)
    for ep in FWD_EPILOGS:
        gpu = run_forward(inp, ep, DT[dtype])
        _expect_variant(gpu["info"], "pair", T)
        check_forward(inp, ep, DT[dtype], gpu)
    fwd = run_forward(inp, "RELU_AUX_BIAS", DT[dtype])
    outs = run_backward(inp, fwd["aux"], DT[dtype], repeats=2)
    for gpu in outs:
        _expect_variant(gpu["info"], "pair", T)
        check_backward(inp, fwd["aux"], DT[dtype], gpu)
    assert torch.equal(outs[0]["dbias"], outs[1]["dbias"])
    for ep in FWD_EPILOGS:
        check_forward(inp, ep, DT[dtype], run_forward(inp, ep, DT[dtype], unfused=True), stored_xw=True)


# The bias gradient's finishing pass over more than 16 row blocks with a
# partial batch last (T = 2300: 18 blocks of 128 rows) and a ragged last
# column tile (N = 776), for each layout of its tickets: 128 or 256 columns
# per ticket on one-CTA tiles, two 128-column tickets per CTA-pair tile.
@pytest.mark.parametrize("variant", ["tile128", "tile256", "pair"])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_dbias_finish_over_many_row_blocks(monkeypatch, dtype, variant):
    _force(monkeypatch, variant)
    T, N, K, D2 = 2300, 776, 64, 136
    inp = synth.make_shape_inputs(T, N, K, dtype, seed=T + N, D2=D2)
    fwd = run_forward(inp, "RELU_AUX_BIAS", DT[dtype])
    outs = run_backward(inp, fwd["aux"], DT[dtype], repeats=2)  # tickets reset between launches
    for gpu in outs:
        _expect_variant(gpu["info"], variant, T)
        check_backward(inp, fwd["aux"], DT[dtype], gpu)
    assert torch.equal(outs[0]["dbias"], outs[1]["dbias"])
    iinp = synth.make_shape_inputs(T, N, K, dtype, seed=T + N + 1, D2=D2, kind="int")
    ifwd = run_forward(iinp, "RELU_AUX_BIAS", DT[dtype])
    check_backward(iinp, ifwd["aux"], DT[dtype], run_backward(iinp, ifwd["aux"], DT[dtype]), exact=True)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("T,N,K", SKINNY_SHAPES)
def test_skinny_split_tiles(monkeypatch, T, N, K, dtype):
    """Few-row kernel on shapes whose tiles are shared by several CTAs (T = 256
    forced onto it: the planner gives 129 rows and more to the tile kernels)."""
    monkeypatch.delenv("GEMM_EPI_FORCE_KERNEL", raising=False)
    if T > 128:
        monkeypatch.setenv("GEMM_EPI_FORCE_KERNEL", "skinny")
    D2 = K
    inp = synth.make_shape_inputs(T, N, K, dtype, seed=T + N + K, D2=D2)
    for ep in FWD_EPILOGS:
        gpu = run_forward(inp, ep, DT[dtype])
        assert gpu["info"]["kernel"] == 1
        check_forward(inp, ep, DT[dtype], gpu)
    fwd = run_forward(inp, "RELU_AUX_BIAS", DT[dtype])
    outs = run_backward(inp, fwd["aux"], DT[dtype], repeats=2)  # tickets reset between launches
    for gpu in outs:
        assert gpu["info"]["kernel"] == 1
        check_backward(inp, fwd["aux"], DT[dtype], gpu)
    assert torch.equal(outs[0]["dbias"], outs[1]["dbias"])


@pytest.mark.parametrize("variant", ["tile128", "pair"])
@pytest.mark.parametrize("raster,group", [("n", 1), ("n", 3), ("m", 2)])
def test_raster_orders(monkeypatch, variant, raster, group):
    """Tile order by column groups (W's block held in L2, X streamed) and small
    row groups: every tile is computed exactly once whatever the order
    (ragged T and N, more tiles than CTAs, DRELU_BGRAD tickets included)."""
    _force(monkeypatch, variant)
    monkeypatch.setenv("GEMM_EPI_RASTER", raster)
    monkeypatch.setenv("GEMM_EPI_GROUP_M", str(group))
    T, N, K = 1800, 3000, 72
    inp = synth.make_shape_inputs(T, N, K, "bf16", seed=61 + group, D2=40)
    for ep in ("RELU_AUX_BIAS", "GELU_AUX_BIAS"):
        gpu = run_forward(inp, ep, torch.bfloat16)
        _expect_variant(gpu["info"], variant, T)
        check_forward(inp, ep, torch.bfloat16, gpu)
    fwd = run_forward(inp, "RELU_AUX_BIAS", torch.bfloat16)
    outs = run_backward(inp, fwd["aux"], torch.bfloat16, repeats=2)
    for gpu in outs:
        check_backward(inp, fwd["aux"], torch.bfloat16, gpu)
    assert torch.equal(outs[0]["dbias"], outs[1]["dbias"])


# CTA pairs in stream-K mode (fewer 256 x 256 tiles than pairs, K of at least
# 16 k-blocks): tiles split over 2 to 9 pairs, ragged T and N, rows of the
# peer CTA past T
PAIR_SPLIT_SHAPES = [(300, 520, 2048), (200, 1032, 1024), (1000, 264, 4096), (256, 2056, 1096)]


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("T,N,K", PAIR_SPLIT_SHAPES)
def test_pair_stream_k(monkeypatch, T, N, K, dtype):
    """Every epilog and DRELU_BGRAD (twice: the segment counters start from
    zero again) through the CTA-pair kernel's stream-K mode; the unfused GEMM
    and integer inputs (bit-exact whatever the split) too."""
    _force(monkeypatch, "pair")
    monkeypatch.setenv("GEMM_EPI_PAIR_SPLIT", "1")
    inp = synth.make_shape_inputs(T, N, K, dtype, seed=T + 5 * N + K, D2=K)
    for ep in FWD_EPILOGS:
        gpu = run_forward(inp, ep, DT[dtype])
        assert gpu["info"]["kernel"] == 2 and gpu["info"]["split_k"] > 1, gpu["info"]
        check_forward(inp, ep, DT[dtype], gpu)
    fwd = run_forward(inp, "RELU_AUX_BIAS", DT[dtype])
    outs = run_backward(inp, fwd["aux"], DT[dtype], repeats=2)
    for gpu in outs:
        assert gpu["info"]["split_k"] > 1
        check_backward(inp, fwd["aux"], DT[dtype], gpu)
    assert torch.equal(outs[0]["dbias"], outs[1]["dbias"])
    assert torch.equal(outs[0]["dZ"].view(torch.int16), outs[1]["dZ"].view(torch.int16))
    check_forward(inp, "RELU_BIAS", DT[dtype], run_forward(inp, "RELU_BIAS", DT[dtype], unfused=True), stored_xw=True)
    iinp = synth.make_shape_inputs(T, N, K, dtype, seed=T + N, D2=K, kind="int")
    check_forward(iinp, "RELU_AUX_BIAS", DT[dtype], run_forward(iinp, "RELU_AUX_BIAS", DT[dtype]), exact=True)
    ifwd = run_forward(iinp, "RELU_AUX_BIAS", DT[dtype])
    check_backward(iinp, ifwd["aux"], DT[dtype], run_backward(iinp, ifwd["aux"], DT[dtype]), exact=True)


# stream-K over at least one wave of tiles: every k-range spans a tile or
# more, so a tile has at most two segments; the second shape keeps one
# data-parallel round of whole tiles, after the stream-K tiles (their
# finishing segments read the other's partial from global memory while the
# next tile's MMAs run) or before them (the pair's last unit brings it in
# with bulk copies)
@pytest.mark.parametrize("sk_first", ["1", "0"])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("T,N,K", [(1024, 4864, 1024), (1100, 9728, 1024)])
def test_pair_stream_k_waves(monkeypatch, T, N, K, dtype, sk_first):
    _force(monkeypatch, "pair")
    monkeypatch.setenv("GEMM_EPI_PAIR_SPLIT", "1")
    monkeypatch.setenv("GEMM_EPI_PAIR_SK_FIRST", sk_first)
    inp = synth.make_shape_inputs(T, N, K, dtype, seed=T + N + 3 * K, D2=K)
    for ep in ("RELU_AUX_BIAS", "GELU_AUX_BIAS"):
        gpu = run_forward(inp, ep, DT[dtype])
        assert gpu["info"]["kernel"] == 2 and gpu["info"]["split_k"] == 2, gpu["info"]
        check_forward(inp, ep, DT[dtype], gpu)
    fwd = run_forward(inp, "RELU_AUX_BIAS", DT[dtype])
    outs = run_backward(inp, fwd["aux"], DT[dtype], repeats=2)
    for gpu in outs:
        check_backward(inp, fwd["aux"], DT[dtype], gpu)
    assert torch.equal(outs[0]["dbias"], outs[1]["dbias"])
    assert torch.equal(outs[0]["dZ"].view(torch.int16), outs[1]["dZ"].view(torch.int16))
    if T == 1024:
        iinp = synth.make_shape_inputs(T, N, K, dtype, seed=T + N, D2=K, kind="int")
        check_forward(iinp, "BIAS", DT[dtype], run_forward(iinp, "BIAS", DT[dtype]), exact=True)


def test_pair_whole_tiles_by_default_when_the_last_round_is_thin(monkeypatch):
    """80 pair tiles for 74 pairs: the last round holds 12 half tiles, and the
    planner keeps whole tiles (stream-K is opt-in)."""
    for k in ("GEMM_EPI_FORCE_KERNEL", "GEMM_EPI_PAIR_SPLIT", "GEMM_EPI_FORCE_BN"):
        monkeypatch.delenv(k, raising=False)
    T, N, K = 1024, 5120, 1024
    inp = synth.make_shape_inputs(T, N, K, "bf16", seed=9, D2=K)
    gpu = run_forward(inp, "RELU_AUX_BIAS", torch.bfloat16)
    assert gpu["info"]["kernel"] == 2 and gpu["info"]["split_k"] == 1, gpu["info"]
    check_forward(inp, "RELU_AUX_BIAS", torch.bfloat16, gpu)
    out = run_backward(inp, gpu["aux"], torch.bfloat16)
    check_backward(inp, gpu["aux"], torch.bfloat16, out)


def test_pair_stream_k_is_off_by_default(monkeypatch):
    _force(monkeypatch, "pair")
    monkeypatch.delenv("GEMM_EPI_PAIR_SPLIT", raising=False)
    T, N, K = 300, 520, 2048
    inp = synth.make_shape_inputs(T, N, K, "bf16", seed=5, D2=K)
    gpu = run_forward(inp, "RELU_AUX_BIAS", torch.bfloat16)
    assert gpu["info"]["kernel"] == 2 and gpu["info"]["split_k"] == 1
    check_forward(inp, "RELU_AUX_BIAS", torch.bfloat16, gpu)


# k per pipeline stage (64·KPS): K ragged against 128, K below one k-block
# (a stage's second 64-k box wholly past K), stream-K segments
KPS_SHAPES = [(1, 1032, 200), (16, 1032, 72), (40, 264, 40), (64, 2056, 1000), (128, 1032, 520), (33, 11008, 1096)]


@pytest.mark.parametrize("kps", [1, 2])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("T,N,K", KPS_SHAPES)
def test_skinny_stage_depth(monkeypatch, T, N, K, dtype, kps):
    """Few-row kernel with 1 or 2 k-blocks per stage, every epilog."""
    monkeypatch.setenv("GEMM_EPI_FORCE_KERNEL", "skinny")
    monkeypatch.setenv("GEMM_EPI_SKINNY_KPS", str(kps))
    D2 = max(8, K // 8 * 8 + 8)
    inp = synth.make_shape_inputs(T, N, K, dtype, seed=11 * T + N + K + kps, D2=D2)
    for ep in FWD_EPILOGS:
        gpu = run_forward(inp, ep, DT[dtype])
        assert gpu["info"]["kernel"] == 1
        assert gpu["info"]["tile_k"] == 64 * kps
        check_forward(inp, ep, DT[dtype], gpu)
    fwd = run_forward(inp, "RELU_AUX_BIAS", DT[dtype])
    outs = run_backward(inp, fwd["aux"], DT[dtype], repeats=2)
    for gpu in outs:
        check_backward(inp, fwd["aux"], DT[dtype], gpu)
    assert torch.equal(outs[0]["dbias"], outs[1]["dbias"])


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("T,N,K,D2", [(130, 72, 64, 40), (257, 520, 128, 96), (64, 8, 8, 8), (16, 1032, 1024, 512),
                                      (300, 1024, 64, 40)])
@pytest.mark.parametrize("variant", ["auto", "pair"])
def test_integer_inputs_bit_exact(monkeypatch, T, N, K, D2, dtype, variant):
    """Integer inputs: every sum is exact in fp32, so Y, aux, dZ and dbias
    must equal the exact result rounded once (pins ties Z == 0, the mask
    layout and the backward operand orientation)."""
    if variant == "pair":
        _force(monkeypatch, "pair")
    inp = synth.make_shape_inputs(T, N, K, dtype, seed=900 + T, D2=D2, kind="int")
    for ep in FWD_EPILOGS:
        gpu = run_forward(inp, ep, DT[dtype])
        check_forward(inp, ep, DT[dtype], gpu, exact=True)
    fwd = run_forward(inp, "RELU_AUX_BIAS", DT[dtype])
    gpu = run_backward(inp, fwd["aux"], DT[dtype])
    check_backward(inp, fwd["aux"], DT[dtype], gpu, exact=True)


def test_zero_bias_is_plain_gemm_relu():
    T, N, K = 200, 136, 96
    inp = synth.make_shape_inputs(T, N, K, "fp16", seed=77)
    inp["bias"] = torch.zeros(N, dtype=torch.float16)
    gpu = run_forward(inp, "RELU_BIAS", torch.float16)
    ref = (inp["X"].double() @ inp["W"].double()).clamp_min(0)
    S = (inp["X"].double().abs() @ inp["W"].double().abs())
    assert torch.all((gpu["Y"].double() - ref).abs() <= 2e-3 * S)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_unfused_path_matches_oracle(dtype):
    T, N, K, D2 = 257, 264, 200, 136
    inp = synth.make_shape_inputs(T, N, K, dtype, seed=31, D2=D2)
    for ep in FWD_EPILOGS:
        gpu = run_forward(inp, ep, DT[dtype], unfused=True)
        check_forward(inp, ep, DT[dtype], gpu, stored_xw=True)
    fwd = run_forward(inp, "RELU_AUX_BIAS", DT[dtype])
    gpu = run_backward(inp, fwd["aux"], DT[dtype], unfused=True)
    check_backward(inp, fwd["aux"], DT[dtype], gpu, stored_dz=True)


def test_dbias_bitwise_reproducible_across_runs_and_streams():
    T, N, D2 = 1000, 520, 264
    inp = synth.make_shape_inputs(T, N, 64, "bf16", seed=5, D2=D2)
    fwd = run_forward(inp, "RELU_AUX_BIAS", torch.bfloat16)
    outs = run_backward(inp, fwd["aux"], torch.bfloat16, repeats=3)
    for o in outs[1:]:
        assert torch.equal(o["dbias"], outs[0]["dbias"])
        assert torch.equal(o["dZ"].view(torch.int16), outs[0]["dZ"].view(torch.int16))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        other = run_backward(inp, fwd["aux"], torch.bfloat16)
    s.synchronize()
    assert torch.equal(other["dbias"], outs[0]["dbias"])


def test_few_row_kernel_only_where_its_32_bit_ranges_fit(monkeypatch):
    """The few-row kernel's range arithmetic is 32-bit, so the planner gives
    it a few-row shape only while (64-deep k-blocks + 1) x SMs stays below
    2^31; a legal shape beyond that (N = K = 2^20: 2^27 k-blocks) goes to the
    tile kernel. Planning only: nothing of that size is allocated or run."""
    monkeypatch.delenv("GEMM_EPI_FORCE_KERNEL", raising=False)
    with binding.Plan(1, 11008, 4096, torch.bfloat16, "RELU_BIAS") as small:
        assert small.info()["kernel"] == 1
    with binding.Plan(1, 1 << 20, 1 << 20, torch.bfloat16, "RELU_BIAS") as huge:
        assert huge.info()["kernel"] == 0


def test_plan_reuse_many_executes():
    """One plan, several executes with different buffers (tensor maps re-encoded)."""
    T, N, K = 300, 264, 136
    with binding.Plan(T, N, K, torch.float16, "RELU_AUX_BIAS") as plan:
        for seed in (1, 2, 3):
            inp = synth.make_shape_inputs(T, N, K, "fp16", seed=seed)
            g = {k: v.cuda() for k, v in inp.items()}
            Y, aux = plan.forward(g["X"], g["W"], g["bias"])
            torch.cuda.synchronize()
            check_forward(inp, "RELU_AUX_BIAS", torch.float16,
                          {"Y": Y.cpu(), "aux": aux.cpu().numpy().view(np.uint32)})


def test_error_paths_on_device():
    T, N, K = 64, 64, 64
    dev = "cuda"
    X = torch.zeros(T * K + 8, dtype=torch.float16, device=dev)
    W = torch.zeros(K, N, dtype=torch.float16, device=dev)
    b = torch.zeros(N, dtype=torch.float16, device=dev)
    Y = torch.zeros(T, N, dtype=torch.float16, device=dev)
    L = binding.lib()
    h = binding.gemm_epi_plan(T, N, K, binding.F16, binding.RELU_AUX_BIAS)
    try:
        s = torch.cuda.current_stream().cuda_stream
        # misaligned X (2-byte offset)
        rc = L.gemm_epi_execute(h, X.data_ptr() + 2, W.data_ptr(), b.data_ptr(), Y.data_ptr(), Y.data_ptr(), s)
        assert rc == binding.ERR_MISALIGNED
        # RELU_AUX_BIAS without aux
        rc = L.gemm_epi_execute(h, X.data_ptr(), W.data_ptr(), b.data_ptr(), Y.data_ptr(), None, s)
        assert rc == binding.ERR_EPILOG_MISMATCH
        # backward call on a forward plan
        rc = L.drelu_bgrad_execute(h, X.data_ptr(), W.data_ptr(), Y.data_ptr(), Y.data_ptr(), Y.data_ptr(), s)
        assert rc == binding.ERR_EPILOG_MISMATCH
        # NULL bias
        rc = L.gemm_epi_execute(h, X.data_ptr(), W.data_ptr(), None, Y.data_ptr(), Y.data_ptr(), s)
        assert rc == binding.ERR_INVALID_ARG
    finally:
        binding.gemm_epi_free(h)
    binding.gemm_epi_free(h)  # double free is ignored
    assert L.gemm_epi_execute(h, X.data_ptr(), W.data_ptr(), b.data_ptr(), Y.data_ptr(), Y.data_ptr(),
                              None) == binding.ERR_INVALID_ARG
    hb = binding.gemm_epi_plan(T, N, K, binding.F16, binding.DRELU_BGRAD)
    try:
        rc = L.gemm_epi_execute(hb, X.data_ptr(), W.data_ptr(), b.data_ptr(), Y.data_ptr(), Y.data_ptr(), None)
        assert rc == binding.ERR_EPILOG_MISMATCH
    finally:
        binding.gemm_epi_free(hb)


@pytest.mark.parametrize("variant", ["tile128", "tile256", "skinny", "pair"])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("T,N,K", [(200, 264, 136), (16, 1032, 520), (600, 1024, 328)])
def test_fp32_bias(monkeypatch, T, N, K, dtype, variant):
    """Forward epilogs with an fp32 bias (values no 16-bit type holds), fused and unfused."""
    _force(monkeypatch, variant)
    inp = synth.make_shape_inputs(T, N, K, dtype, seed=17 * T + N + K)
    inp["bias32"] = synth.normal((N,), synth.BIAS_STD, torch.float32, seed=T + 2 * N)
    for ep in FWD_EPILOGS:
        gpu = run_forward(inp, ep, DT[dtype], bias_f32=True)
        check_forward(inp, ep, DT[dtype], gpu, bias_f32=True)
        gpu = run_forward(inp, ep, DT[dtype], bias_f32=True, unfused=True)
        check_forward(inp, ep, DT[dtype], gpu, bias_f32=True, stored_xw=True)


# weight given N x K (a framework linear layer's [out, in] layout): ragged
# shapes, one with more than a wave of CTA pairs (no half tiles then)
NK_SHAPES = [(200, 264, 136), (16, 1032, 520), (600, 1024, 328), (1000, 5000, 72)]


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("T,N,K", NK_SHAPES)
def test_weight_nk_layout(monkeypatch, T, N, K, dtype, variant):
    _force(monkeypatch, variant)
    D2 = max(8, (K // 2) // 8 * 8)
    inp = synth.make_shape_inputs(T, N, K, dtype, seed=13 * T + N + 3 * K, D2=D2)
    for ep in FWD_EPILOGS:
        gpu = run_forward(inp, ep, DT[dtype], w_nk=True)
        assert gpu["info"]["kernel"] != 1  # an N x K weight never runs on the few-row kernel
        check_forward(inp, ep, DT[dtype], gpu)
    check_forward(inp, "RELU_BIAS", DT[dtype], run_forward(inp, "RELU_BIAS", DT[dtype], w_nk=True, unfused=True),
                  stored_xw=True)
    fwd = run_forward(inp, "RELU_AUX_BIAS", DT[dtype])
    outs = run_backward(inp, fwd["aux"], DT[dtype], w_nk=True, repeats=2)
    for gpu in outs:
        assert gpu["info"]["kernel"] != 1
        check_backward(inp, fwd["aux"], DT[dtype], gpu)
    assert torch.equal(outs[0]["dbias"], outs[1]["dbias"])


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("variant", ["auto", "pair"])
def test_weight_nk_integer_inputs_bit_exact(monkeypatch, dtype, variant):
    if variant == "pair":
        _force(monkeypatch, "pair")
    T, N, K, D2 = 300, 1024, 64, 40
    inp = synth.make_shape_inputs(T, N, K, dtype, seed=77, D2=D2, kind="int")
    for ep in ("BIAS", "RELU_AUX_BIAS"):
        check_forward(inp, ep, DT[dtype], run_forward(inp, ep, DT[dtype], w_nk=True), exact=True)
    fwd = run_forward(inp, "RELU_AUX_BIAS", DT[dtype])
    check_backward(inp, fwd["aux"], DT[dtype], run_backward(inp, fwd["aux"], DT[dtype], w_nk=True), exact=True)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("T,D,F", [(256, 136, 264), (300, 512, 1032), (64, 128, 200)])
def test_ffn_step_chain_bit_exact(T, D, F, dtype):
    """A whole two-layer block step, six library calls chained on integer
    inputs: every intermediate and output equals the oracle's exact value
    (rounded once to the 16-bit type where the step stores it)."""
    inp = synth.ffn_step_inputs(T, D, F, dtype, seed=T + D + F, kind="int")
    bits = {k: synth.bits_u16(v) for k, v in inp.items()}
    dt = DT[dtype]
    ref = oracle.ffn_step(bits["X"], bits["W1"], bits["b1"], bits["W2"], bits["b2"], bits["dY"], odt(dt))
    gpu = run_ffn_step(inp, dt)
    for k in ("H", "Y", "dZ1", "dW2", "dW1", "dX"):
        expect = torch.from_numpy(ref[k]).to(dt)
        assert torch.equal(gpu[k].view(torch.int16), expect.view(torch.int16)), f"{k} differs"
    for k in ("db1", "db2"):
        assert np.array_equal(gpu[k].double().numpy(), ref[k]), f"{k} differs"
    assert np.array_equal(oracle.relu_aux_bits(gpu["aux"].numpy().view(np.uint32), F), ref["bits"])


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("T,N,K", [(200, 264, 136), (16, 1032, 520), (600, 1024, 328), (1000, 5000, 72), (5, 40, 24)])
def test_fp32_output(monkeypatch, T, N, K, dtype, variant):
    """16-bit operands, fp32 Y / dZ / dW (GEMM_EPI_FLAG_OUT_F32): the accumulator itself."""
    _force(monkeypatch, variant)
    D2 = max(8, (K // 2) // 8 * 8)
    inp = synth.make_shape_inputs(T, N, K, dtype, seed=19 * T + N + K, D2=D2)
    for ep in FWD_EPILOGS:
        gpu = run_forward(inp, ep, DT[dtype], out_f32=True)
        assert gpu["Y"].dtype == torch.float32
        check_forward(inp, ep, DT[dtype], gpu)
    fwd = run_forward(inp, "RELU_AUX_BIAS", DT[dtype])
    outs = run_backward(inp, fwd["aux"], DT[dtype], out_f32=True, repeats=2)
    for gpu in outs:
        assert gpu["dZ"].dtype == torch.float32
        check_backward(inp, fwd["aux"], DT[dtype], gpu)
    assert torch.equal(outs[0]["dbias"], outs[1]["dbias"])
    if variant != "skinny":
        winp = synth.make_shape_inputs(T, N, K, dtype, seed=T + 7 * N + K, D2=N)
        check_wgrad(winp, DT[dtype], run_wgrad(winp, DT[dtype], out_f32=True))


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_fp32_output_integer_inputs_exact(dtype):
    T, N, K, D2 = 300, 1024, 64, 40
    inp = synth.make_shape_inputs(T, N, K, dtype, seed=78, D2=D2, kind="int")
    for ep in ("BIAS", "RELU_AUX_BIAS"):
        check_forward(inp, ep, DT[dtype], run_forward(inp, ep, DT[dtype], out_f32=True), exact=True)
    fwd = run_forward(inp, "RELU_AUX_BIAS", DT[dtype])
    check_backward(inp, fwd["aux"], DT[dtype], run_backward(inp, fwd["aux"], DT[dtype], out_f32=True), exact=True)


def test_fp32_output_unfused_is_refused():
    h = binding.gemm_epi_plan(64, 64, 64, binding.F16, binding.RELU_BIAS, flags=binding.FLAG_OUT_F32)
    try:
        p = torch.zeros(64 * 64, dtype=torch.float32, device="cuda").data_ptr()
        rc = binding.lib().gemm_epi_unfused_execute(h, p, p, p, p, p, p, None, None)
        assert rc == binding.ERR_UNSUPPORTED
    finally:
        binding.gemm_epi_free(h)


def test_plan_flags_are_checked():
    with pytest.raises(binding.GemmEpiError):
        binding.gemm_epi_plan(64, 64, 64, binding.F16, binding.RELU_BIAS, flags=4)  # no such flag
    with pytest.raises(binding.GemmEpiError):
        binding.gemm_epi_plan(64, 64, 64, binding.F16, binding.WGRAD, flags=binding.FLAG_W_NK)


# weight gradient dW = X^T dZ: ragged K (dW rows), N and T (the contraction),
# T = 1, and enough tiles for more than one wave of CTA pairs
WGRAD_SHAPES = [(200, 264, 136), (1, 72, 64), (130, 520, 328), (1000, 1032, 264), (257, 8, 8), (64, 640, 192),
                (777, 2056, 1104)]


@pytest.mark.parametrize("variant", ["tile64", "tile128", "tile192", "tile256", "pair"])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("T,N,K", WGRAD_SHAPES)
def test_wgrad_matches_oracle(monkeypatch, T, N, K, dtype, variant):
    _force(monkeypatch, variant)
    inp = synth.make_shape_inputs(T, N, K, dtype, seed=3 * T + N + 5 * K, D2=N)
    gpu = run_wgrad(inp, DT[dtype])
    # dW has K rows: the CTA-pair kernel when forced and K > 128, else one CTA per tile (never the few-row kernel)
    assert gpu["info"]["kernel"] == (2 if variant == "pair" and K > 128 else 0)
    assert (gpu["info"]["T"], gpu["info"]["N"], gpu["info"]["K"]) == (T, N, K)
    check_wgrad(inp, DT[dtype], gpu)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("variant", ["auto", "pair"])
def test_wgrad_integer_inputs_bit_exact(monkeypatch, dtype, variant):
    if variant == "pair":
        _force(monkeypatch, "pair")
    T, N, K = 300, 520, 264
    inp = synth.make_shape_inputs(T, N, K, dtype, seed=41, D2=N, kind="int")
    check_wgrad(inp, DT[dtype], run_wgrad(inp, DT[dtype]), exact=True)


def test_wgrad_plan_rejects_other_calls():
    T, N, K = 64, 64, 64
    X = torch.zeros(T, K, dtype=torch.float16, device="cuda")
    L = binding.lib()
    h = binding.gemm_epi_plan(T, N, K, binding.F16, binding.WGRAD)
    try:
        s = torch.cuda.current_stream().cuda_stream
        p = X.data_ptr()
        assert L.gemm_epi_execute(h, p, p, p, p, p, s) == binding.ERR_EPILOG_MISMATCH
        assert L.drelu_bgrad_execute(h, p, p, p, p, p, s) == binding.ERR_EPILOG_MISMATCH
        assert L.gemm_epi_wgrad_execute(h, p + 2, p, p, None, s) == binding.ERR_MISALIGNED
        assert L.gemm_epi_wgrad_execute(h, p, None, p, None, s) == binding.ERR_INVALID_ARG
        assert L.gemm_epi_set_bias_f32(h, 1) == binding.ERR_EPILOG_MISMATCH
        assert L.gemm_epi_wgrad_execute(h, p, p, p, p + 2, s) == binding.ERR_MISALIGNED  # dbias
    finally:
        binding.gemm_epi_free(h)
    hf = binding.gemm_epi_plan(T, N, K, binding.F16, binding.RELU_BIAS)
    try:
        assert L.gemm_epi_wgrad_execute(hf, p, p, p, None, None) == binding.ERR_EPILOG_MISMATCH
    finally:
        binding.gemm_epi_free(hf)


def test_injected_encode_failure_returns_error_without_launch(monkeypatch):
    """A failing tensor-map encode (forced on the host) is reported by execute
    as GEMM_EPI_ERR_CUDA; the output stays untouched (nothing was launched)."""
    T, N, K = 128, 128, 64
    inp = synth.make_shape_inputs(T, N, K, "bf16", seed=2)
    g = {k: v.cuda() for k, v in inp.items()}
    with binding.Plan(T, N, K, torch.bfloat16, "RELU_BIAS") as plan:
        Y = torch.full((T, N), 7.0, dtype=torch.bfloat16, device="cuda")
        monkeypatch.setenv("GEMM_EPI_TEST_HOOKS", "1")
        monkeypatch.setenv("GEMM_EPI_INJECT_ENCODE_FAILURE", "1")
        with pytest.raises(binding.GemmEpiError) as e:
            plan.gemm_epi_execute(g["X"], g["W"], g["bias"], Y)
        assert e.value.code == binding.ERR_CUDA and "injected" in str(e.value)
        torch.cuda.synchronize()
        assert torch.all(Y == 7.0)
        monkeypatch.delenv("GEMM_EPI_INJECT_ENCODE_FAILURE")
        plan.gemm_epi_execute(g["X"], g["W"], g["bias"], Y)  # the plan still works afterwards
        torch.cuda.synchronize()
        assert plan.status() == 0 and not torch.all(Y == 7.0)


def test_unknown_epilog_values_rejected():
    for bad in (-1, 8, 99):
        with pytest.raises(binding.GemmEpiError):
            binding.gemm_epi_plan(64, 64, 64, binding.F16, bad)


def test_injected_workspace_allocation_failure(monkeypatch):
    monkeypatch.setenv("GEMM_EPI_INJECT_PLAN_ALLOC_FAILURE", "1")
    binding.gemm_epi_free(binding.gemm_epi_plan(256, 256, 256, binding.BF16, binding.DRELU_BGRAD))  # hooks off
    monkeypatch.setenv("GEMM_EPI_TEST_HOOKS", "1")
    with pytest.raises(binding.GemmEpiError) as e:
        binding.gemm_epi_plan(256, 256, 256, binding.BF16, binding.DRELU_BGRAD)
    assert "injected" in str(e.value)


# (kernel variant, T, N, K): the one-CTA kernel (BN = 64), the CTA pair (the
# peer's epilogue waits on a commit from the leader and both drain through the
# final cluster barrier; the second shape gives each pair two or three units,
# so the leader's MMA issuer must give up on a later unit; the third runs in
# stream-K mode, where a tile's segment 0 waits on the other segments'
# partials) and the few-row kernel (a tile split into stream-K
# segments, whose tickets must be reset after the abort)
WATCHDOG_CASES = [("tile64", 512, 512, 256), ("pair", 512, 512, 256), ("pair", 2048, 5120, 64),
                  ("pair", 300, 520, 2048), ("skinny", 16, 1032, 2048)]


@pytest.mark.parametrize("variant,T,N,K", WATCHDOG_CASES)
@pytest.mark.parametrize("epilog", ["RELU_AUX_BIAS", "DRELU_BGRAD"])
def test_watchdog_reports_timeout_and_context_stays_usable(monkeypatch, epilog, variant, T, N, K):
    """Fault injection without a GPU fault: the MMA issuer withholds the first
    tile's completion signal, the epilogue's bounded wait (200 ms here) runs
    out, the kernel drains its copies and MMAs, frees its tensor memory and
    returns, and the host reads ERR_TIMEOUT. The same plan and a fresh one
    afterwards must compute correctly."""
    _force(monkeypatch, variant)
    if variant == "pair" and K >= 1024:
        monkeypatch.setenv("GEMM_EPI_PAIR_SPLIT", "1")
    monkeypatch.setenv("GEMM_EPI_WAIT_TIMEOUT_MS", "200")
    monkeypatch.setenv("GEMM_EPI_INJECT_STALL", "1")
    monkeypatch.setenv("GEMM_EPI_TEST_HOOKS", "1")
    inp = synth.make_shape_inputs(T, N, K, "bf16", seed=17, D2=K)
    g = {k: v.cuda() for k, v in inp.items()}
    dt = torch.bfloat16
    aux = torch.zeros((T, (N + 31) // 32), dtype=torch.int32, device="cuda")
    with binding.Plan(T, N, K, dt, epilog) as plan:
        _expect_variant(plan.info(), variant, T)
        if epilog == "DRELU_BGRAD":
            plan.backward(g["dY2"], g["W2"], aux)
        else:
            plan.forward(g["X"], g["W"], g["bias"])
        torch.cuda.synchronize()  # returns: the kernel gave up and exited
        assert plan.status() == binding.ERR_TIMEOUT
        assert "watchdog" in binding.gemm_epi_last_error()
        assert plan.status() == binding.OK  # the report is cleared by reading it
    monkeypatch.delenv("GEMM_EPI_INJECT_STALL")
    gpu = run_forward(inp, "RELU_AUX_BIAS", dt)
    _expect_variant(gpu["info"], variant, T)
    check_forward(inp, "RELU_AUX_BIAS", dt, gpu)
    outs = run_backward(inp, gpu["aux"], dt, repeats=2)  # split-tile and column tickets start from zero again
    for out in outs:
        check_backward(inp, gpu["aux"], dt, out)


@pytest.mark.parametrize("epilog", ["GELU_BIAS", "GELU_AUX_BIAS"])
def test_watchdog_with_eight_epilogue_warps(monkeypatch, epilog):
    """The CTA-pair kernel's GELU instances (two epilogue warps per TMEM lane
    quarter): the same injected stall, the same report, and correct results
    afterwards."""
    _force(monkeypatch, "pair")
    monkeypatch.setenv("GEMM_EPI_WAIT_TIMEOUT_MS", "200")
    monkeypatch.setenv("GEMM_EPI_INJECT_STALL", "1")
    monkeypatch.setenv("GEMM_EPI_TEST_HOOKS", "1")
    T, N, K = 600, 1032, 264
    inp = synth.make_shape_inputs(T, N, K, "bf16", seed=19)
    g = {k: v.cuda() for k, v in inp.items()}
    with binding.Plan(T, N, K, torch.bfloat16, epilog) as plan:
        assert plan.info()["kernel"] == 2
        plan.forward(g["X"], g["W"], g["bias"])
        torch.cuda.synchronize()
        assert plan.status() == binding.ERR_TIMEOUT
    monkeypatch.delenv("GEMM_EPI_INJECT_STALL")
    gpu = run_forward(inp, epilog, torch.bfloat16)
    assert gpu["info"]["kernel"] == 2
    check_forward(inp, epilog, torch.bfloat16, gpu)


def test_stall_hook_needs_the_test_switch(monkeypatch):
    """GEMM_EPI_INJECT_STALL alone (without GEMM_EPI_TEST_HOOKS=1) changes nothing."""
    _force(monkeypatch, "tile64")
    monkeypatch.setenv("GEMM_EPI_WAIT_TIMEOUT_MS", "200")
    monkeypatch.setenv("GEMM_EPI_INJECT_STALL", "1")
    monkeypatch.delenv("GEMM_EPI_TEST_HOOKS", raising=False)
    inp = synth.make_shape_inputs(256, 256, 128, "bf16", seed=23)
    check_forward(inp, "RELU_AUX_BIAS", torch.bfloat16, run_forward(inp, "RELU_AUX_BIAS", torch.bfloat16))


@pytest.mark.parametrize("variant", ["tile128", "tile256", "pair", "skinny"])
def test_gelu_over_a_wide_range_of_z(monkeypatch, variant):
    """X = I and an fp32 output: Y = gelu(W) element by element, for W from
    -12 to 12 and for magnitudes down to 1e-6 of both signs. The epilogue's
    fp32 GELU, 0.5 z (1 + erff(z / sqrt 2)) with CUDA's erff (2 ulp), against
    the exact z * Phi(z): within 5e-7 |z| plus the fp32 rounding of the
    result."""
    from scipy.special import ndtr
    _force(monkeypatch, variant)
    T = K = 256
    N = 1024
    g = torch.Generator().manual_seed(5)
    lin = torch.linspace(-12.0, 12.0, K * N // 2)
    tiny = torch.sign(torch.rand(K * N // 2, generator=g) - 0.5) * 10.0 ** (torch.rand(K * N // 2, generator=g) * 7.1 - 6.0)
    W = torch.cat([lin, tiny]).reshape(K, N).to(torch.bfloat16)
    X = torch.eye(T, K, dtype=torch.bfloat16)
    bias = torch.zeros(N, dtype=torch.bfloat16)
    with binding.Plan(T, N, K, torch.bfloat16, "GELU_BIAS", out_f32=True) as p:
        Y = torch.empty(T, N, dtype=torch.float32, device="cuda")
        p.gemm_epi_execute(X.cuda(), W.cuda(), bias.cuda(), Y)
        torch.cuda.synchronize()
        assert p.status() == 0
        _expect_variant(p.info(), variant, T)
    z = W.double().numpy()
    ref = z * ndtr(z)
    err = np.abs(Y.cpu().double().numpy() - ref)
    bound = 5e-7 * np.abs(z) + 2.0 ** -24 * np.abs(ref) + 1e-37
    assert np.all(err <= bound), f"worst {np.max(err / bound):.3g} of the bound at z = {z.flat[np.argmax(err / bound)]}"
