"""Parity of the tcgen05 INT8 GEMM + dequant kernels with the oracle, through the C ABI:
int32 accumulators and bf16 outputs bit-exact (the bar is 1 bf16 ulp; the epilogue is built
to the oracle's operation order, so 0 is expected and asserted, and the ulp distance is
reported on failure). Both kernels (persistent tile / swap-AB stream-K) are run on the same
shapes, including ragged M, N and K tails, several tiles, and extreme accumulators."""
import numpy as np
import pytest
import torch

import int8_w8a8_quantized_smoothed_b200 as w8
import oracle
from int8_w8a8_quantized_smoothed_b200 import synth
from helpers import bf16_out, bf16_ulp_distance, dev, dev_bf16, host, host_bf16, with_canary

pytestmark = pytest.mark.gpu


def _inputs(M, N, K, seed):
    xq = synth.int8_codes((M, K), seed)
    wq = synth.int8_codes((N, K), seed + 1)
    st = synth.scales(M, seed + 2, 1e-3, 0.5)
    sc = synth.scales(N, seed + 3, 1e-4, 2e-2)
    return xq, st, wq, sc


def _run(xq, st, wq, sc, variant, ctas=0, tile_n=0):
    M, N = xq.shape[0], wq.shape[0]
    y, cy = bf16_out((M, N))
    acc, ca = with_canary((M, N), torch.int32, -7)
    w8.w8a8_gemm_dequant_ex(dev(xq), dev(st), dev(wq), dev(sc), y=y, acc_out=acc,
                            variant=variant, ctas=ctas, tile_n=tile_n)
    torch.cuda.synchronize()
    cy(); ca()
    return host_bf16(y), host(acc)


def _compare(y, acc, y_ref, acc_ref):
    assert np.array_equal(acc, acc_ref), f"{(acc != acc_ref).sum()} accumulators differ"
    d = bf16_ulp_distance(y, y_ref)
    assert d.max() <= 1, f"bf16 differs by up to {d.max()} ulp"
    assert np.array_equal(y, y_ref), f"{(d > 0).sum()} outputs differ by 1 ulp"


DECODE_SHAPES = [(1, 8, 16), (1, 512, 256), (16, 512, 256), (8, 1024, 4096), (3, 136, 400),
                 (33, 1032, 4096), (64, 1024, 14336), (17, 256, 4112), (100, 384, 1024),
                 (256, 264, 512), (129, 128, 256)]


@pytest.mark.parametrize("M,N,K", DECODE_SHAPES)
@pytest.mark.parametrize("ctas", [0, 1, 3, 7])
def test_decode_kernel_bit_exact(M, N, K, ctas):
    # ctas=1: one CTA walks every block whole; 3 and 7: blocks split between CTAs (owner +
    # contributors); 0: one CTA per SM (the launch the benchmark times)
    xq, st, wq, sc = _inputs(M, N, K, seed=M + N + K)
    y_ref, acc_ref = oracle.gemm_dequant(xq, st, wq, sc)
    y, acc = _run(xq, st, wq, sc, variant=2, ctas=ctas)
    _compare(y, acc, y_ref, acc_ref)


@pytest.mark.parametrize("M,N,K", DECODE_SHAPES)
@pytest.mark.parametrize("cluster", [0, 1, 2, 3, 5, 8])
def test_decode_cluster_kernel_bit_exact(M, N, K, cluster):
    # K split over a thread-block cluster of `cluster` CTAs per 128-channel block; partials
    # summed in distributed shared memory (0: automatic size)
    xq, st, wq, sc = _inputs(M, N, K, seed=2 * M + N + K)
    y_ref, acc_ref = oracle.gemm_dequant(xq, st, wq, sc)
    y, acc = _run(xq, st, wq, sc, variant=3, ctas=cluster)
    _compare(y, acc, y_ref, acc_ref)


# beyond 256 tokens the swap-AB kernels take the tokens in tiles of 256 (ragged last tile)
MULTI_TILE_SHAPES = [(300, 512, 1024), (512, 384, 4096), (777, 1024, 512), (1024, 256, 2048)]


@pytest.mark.parametrize("M,N,K", MULTI_TILE_SHAPES)
@pytest.mark.parametrize("variant,ctas", [(2, 0), (2, 5), (3, 0), (3, 3)])
def test_decode_kernels_multi_token_tile_bit_exact(M, N, K, variant, ctas):
    xq, st, wq, sc = _inputs(M, N, K, seed=5 * M + N + K)
    y_ref, acc_ref = oracle.gemm_dequant(xq, st, wq, sc)
    y, acc = _run(xq, st, wq, sc, variant=variant, ctas=ctas)
    _compare(y, acc, y_ref, acc_ref)


PREFILL_SHAPES = [(1, 8, 16), (16, 512, 256), (128, 256, 128), (129, 264, 400), (200, 136, 208),
                  (300, 1024, 4096), (512, 2048, 1024), (257, 520, 14336), (1000, 3000, 64)]


@pytest.mark.parametrize("M,N,K", PREFILL_SHAPES)
@pytest.mark.parametrize("tile_n", [128, 256, 512])
def test_prefill_kernel_bit_exact(M, N, K, tile_n):
    # tile_n 128 / 256: 128-row tiles, double-buffered accumulators; 512: 256 x 256 tiles
    xq, st, wq, sc = _inputs(M, N, K, seed=3 * M + N + K)
    y_ref, acc_ref = oracle.gemm_dequant(xq, st, wq, sc)
    y, acc = _run(xq, st, wq, sc, variant=1, tile_n=tile_n)
    _compare(y, acc, y_ref, acc_ref)


def test_persistent_kernel_many_tiles_per_cta():
    # more tiles than SMs: every CTA loops over several tiles and both TMEM accumulators
    M, N, K = 2048, 4096, 256
    xq, st, wq, sc = _inputs(M, N, K, 5)
    y_ref, acc_ref = oracle.gemm_dequant(xq, st, wq, sc)
    for tn in (128, 256, 512):
        y, acc = _run(xq, st, wq, sc, variant=1, tile_n=tn)
        _compare(y, acc, y_ref, acc_ref)


def test_extreme_accumulators():
    # |acc| = 127 * 127 * K for K = 14336 (about 2.3e8 > 2^24): int->float rounding matters
    M, N, K = 4, 16, 14336
    xq = np.full((M, K), 127, np.int8)
    xq[1] = -127
    wq = np.full((N, K), 127, np.int8)
    wq[3] = -127
    st = synth.scales(M, 1)
    sc = synth.scales(N, 2)
    y_ref, acc_ref = oracle.gemm_dequant(xq, st, wq, sc)
    assert acc_ref[0, 0] == 127 * 127 * K
    for variant in (1, 2, 3):
        y, acc = _run(xq, st, wq, sc, variant=variant)
        _compare(y, acc, y_ref, acc_ref)


@pytest.mark.parametrize("variant", [1, 2, 3])
def test_largest_k_accumulators_near_int32_limit(variant):
    # K = 133136, the largest multiple of 16 within the library's bound (127^2 K < 2^31):
    # every product is +-127*127 and the sums come within 2^22 of the int32 limit, in the
    # tile kernel, across stream-K CTAs and across an 8-CTA cluster
    M, N, K = 3, 16, 133136
    xq = np.full((M, K), 127, np.int8)
    xq[1] = -127
    xq[2, ::2] = -127
    wq = np.full((N, K), 127, np.int8)
    wq[5] = -127
    st = synth.scales(M, 3)
    sc = synth.scales(N, 4)
    y_ref, acc_ref = oracle.gemm_dequant(xq, st, wq, sc)
    top = int(acc_ref[0, 0])
    assert top == 127 * 127 * K and 2 ** 31 - top < 2 ** 22
    y, acc = _run(xq, st, wq, sc, variant=variant)
    _compare(y, acc, y_ref, acc_ref)


def test_auto_variant_and_workspace_reuse():
    # the stream-K workspace must come back ready for the next call (flags zero): run twice
    # through one workspace, with the automatic choice and forced stream-K
    for (M, N, K) in [(8, 6144, 4096), (64, 4096, 4096), (512, 1024, 1024), (8, 28672, 4096)]:
        xq, st, wq, sc = _inputs(M, N, K, 11)
        y_ref, acc_ref = oracle.gemm_dequant(xq, st, wq, sc)
        ws = w8.Workspace()
        for _ in range(2):
            y = w8.w8a8_gemm_dequant(dev(xq), dev(st), dev(wq), dev(sc), workspace=ws)
            torch.cuda.synchronize()
            assert np.array_equal(host_bf16(y), y_ref)
        for _ in range(2):
            y = w8.w8a8_gemm_dequant_ex(dev(xq), dev(st), dev(wq), dev(sc), workspace=ws,
                                        variant=2 if M <= 256 else 1)
            torch.cuda.synchronize()
            assert np.array_equal(host_bf16(y), y_ref)


def test_zero_scales_give_zero():
    M, N, K = 8, 64, 256
    xq, st, wq, sc = _inputs(M, N, K, 13)
    st[2] = 0.0
    sc[5] = 0.0
    y_ref, _ = oracle.gemm_dequant(xq, st, wq, sc)
    for variant in (1, 2, 3):
        y = w8.w8a8_gemm_dequant_ex(dev(xq), dev(st), dev(wq), dev(sc), variant=variant)
        yh = host_bf16(y)
        assert np.array_equal(yh, y_ref)
        assert not (yh[2] & 0x7FFF).any() and not (yh[:, 5] & 0x7FFF).any()


def test_workspace_too_small_is_reported():
    M, N, K = 8, 1024, 4096
    xq, st, wq, sc = _inputs(M, N, K, 1)
    need = w8.w8a8_gemm_workspace_size_ex(M, N, K, 2, 7, 0)
    assert need > 0
    small = torch.zeros(need - 4, dtype=torch.uint8, device="cuda")
    with pytest.raises(w8.W8A8Error, match="WORKSPACE"):
        w8.w8a8_gemm_dequant_ex(dev(xq), dev(st), dev(wq), dev(sc), workspace=small, variant=2,
                                ctas=7)
    assert w8.w8a8_device_status(reset=True) == 0


def _chain(layers, ws):
    """rmsnorm+quant -> GEMM -> SiLU*up+quant -> GEMM, per layer, with no host sync."""
    outs = []
    for L in layers:
        q, s = w8.w8a8_smooth_rmsnorm_quant(L["x"], L["g"], 1e-5)
        gu = w8.w8a8_gemm_dequant(q, s, *L["w1"], workspace=ws)
        q2, s2 = w8.w8a8_silu_mul_quant(gu)
        outs.append(w8.w8a8_gemm_dequant(q2, s2, *L["w2"], workspace=ws))
    return outs


@pytest.mark.parametrize("M", [1, 33, 300])
def test_overlap_modes_give_identical_results(M):
    # modes 0/1/2 only change when kernels may start; every output must be the same bits,
    # eagerly and when the chain is replayed from a CUDA graph
    H, I = 512, 1024
    layers = []
    for i in range(3):
        layers.append(dict(
            x=dev_bf16(synth.activation(M, H, 10 + i)),
            g=dev(synth.gamma(H, 20 + i)),
            w1=(dev(synth.int8_codes((2 * I, H), 30 + i)), dev(synth.scales(2 * I, 40 + i))),
            w2=(dev(synth.int8_codes((H, I), 50 + i)), dev(synth.scales(H, 60 + i)))))
    torch.cuda.synchronize()
    ws = w8.Workspace()
    prev = w8.w8a8_get_overlap()
    try:
        results = {}
        for mode in (0, 1, 2):
            w8.w8a8_set_overlap(mode)
            eager = [host_bf16(t) for t in _chain(layers, ws)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                outs = _chain(layers, ws)
            for _ in range(3):
                g.replay()
            torch.cuda.synchronize()
            results[mode] = (eager, [host_bf16(t) for t in outs])
            del g
        for mode in (0, 1, 2):
            for a, b in zip(results[0][0] + results[0][1], results[mode][0] + results[mode][1]):
                assert np.array_equal(a, b)
    finally:
        w8.w8a8_set_overlap(prev)
    assert w8.w8a8_device_status(reset=True) == 0


# Stream-K on the CTA-pair tile kernel (variant 1, tile_n 512, ctas = pairs): tiles split
# between pairs are finished by the pair holding their first k-blocks after adding up to three
# later pieces staged through its idle ring. Pair counts that leave 1..3 contributors per
# tile, pairs with empty shares (tiny K), ragged M, N and K tails, and repeated calls on one
# workspace (the owners lower the contributors' flags).
PAIR_SK_CASES = [(300, 1000, 512, 24), (300, 1000, 512, 5), (257, 264, 4112, 5),
                 (512, 4096, 4096, 74), (512, 4096, 14336, 74), (512, 6144, 4096, 74),
                 (129, 264, 16, 6), (520, 256, 1024, 9), (65, 512, 4096, 6),
                 (1000, 4096, 256, 74), (600, 1032, 1040, 37), (256, 256, 384, 3)]


@pytest.mark.parametrize("M,N,K,pairs", PAIR_SK_CASES)
def test_pair_stream_k_bit_exact(M, N, K, pairs):
    xq, st, wq, sc = _inputs(M, N, K, seed=M + 2 * N + K)
    y_ref, acc_ref = oracle.gemm_dequant(xq, st, wq, sc)
    for _ in range(2):
        y, acc = _run(xq, st, wq, sc, variant=1, ctas=pairs, tile_n=512)
        _compare(y, acc, y_ref, acc_ref)
    assert w8.w8a8_device_status(reset=True) == 0


def test_pair_stream_k_is_the_plan_for_few_long_tiles():
    # the M = 512 decoder block's down projection: 32 tiles of 112 k-blocks on 74 pairs
    assert w8.w8a8_gemm_workspace_size(512, 4096, 14336) > 0
    # short tiles, or tiles that fill the pairs, keep the whole-tile schedules
    assert w8.w8a8_gemm_workspace_size(512, 6144, 4096) == 0
    assert w8.w8a8_gemm_workspace_size(8192, 28672, 4096) == 0
