"""GPU parity of the inference product from the stored form (itwiki "GPTQ",
"결과"; blog section 5): gptq_dequant_gemv against oracle.dequant_gemv.

Tolerance: every product c * x is exact and each 128-column block is summed
and scaled in fp32, so |y - y_ref| <= TOL * sum_k |s (c - z) x| per output
(the fp32 accumulation bound, with margin).  A single code off by one level
moves y by s |x_k|, far above it."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_05_b200 import api, build_lib, synth
from parity_util import to_dev_x

pytestmark = pytest.mark.gpu

TOL = 2e-6


@pytest.fixture(scope="module", autouse=True)
def _ready():
    build_lib.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    api.get_status(raise_on_error=False)
    yield
    code, _ = api.get_status(raise_on_error=False)
    assert code == 0


def _stored_form(d_out, d_in, g, seed):
    """Uniform random 4-bit codes (uniform random words), fp16 scales, and
    integer zero points, some of them far outside the code range."""
    rng = np.random.default_rng(seed)
    words = rng.integers(0, 2 ** 32, size=(d_out, d_in // 8), dtype=np.uint64).astype(np.uint32)
    ng = 1 if g <= 0 else d_in // g
    s = (np.abs(rng.standard_normal((d_out, ng))) * 3e-3 + 1e-4).astype(np.float16)
    z = rng.integers(0, 16, size=(d_out, ng)).astype(np.float16)
    z[::7, 0] = -75.0
    z[3::11, -1] = 40.0
    return words, s, z


def _tokens(m, d_in, seed):
    rng = np.random.default_rng(seed + 1)
    xf = rng.standard_normal((m, d_in)).astype(np.float32) * np.exp(rng.normal(0, 1.0, d_in)).astype(np.float32)
    bits = synth.f32_to_bf16_bits(xf)
    return bits, synth.bf16_bits_to_f32(bits)


def _dev(words, s, z, xbits):
    return (torch.from_numpy(words.view(np.int32)).cuda(), torch.from_numpy(s).cuda(), torch.from_numpy(z).cuda(),
            torch.from_numpy(xbits.view(np.int16)).cuda().view(torch.bfloat16))


def _run(words, s, z, g, xbits, perm=None):
    codes, sd, zd, xd = _dev(words, s, z, xbits)
    y = torch.full((xbits.shape[0], words.shape[0]), 123.0, dtype=torch.float32, device="cuda")
    pd = None if perm is None else torch.from_numpy(np.asarray(perm, dtype=np.int32)).cuda()
    api.dequant_gemv(codes, sd, zd, 4, g, xd, y, perm=pd)
    api.get_status()
    return y.cpu().numpy().astype(np.float64)


def _check(y, words, s, z, g, xf, perm=None, rows=None):
    if rows is not None:
        words, s, z, y = words[rows], s[rows], z[rows], y[:, rows]
    s64, z64, x64 = s.astype(np.float64), z.astype(np.float64), xf.astype(np.float64)
    ref = oracle.dequant_gemv(words, s64, z64, 4, g, x64, perm)
    d_in = xf.shape[1]
    gi = np.arange(d_in) // (d_in if g <= 0 else g)
    Qabs = np.abs(oracle.dequant(oracle.unpack_codes(words, 4, d_in), s64[:, gi], z64[:, gi]))
    xp = x64 if perm is None else x64[:, np.asarray(perm)]
    bound = TOL * (np.abs(xp) @ Qabs.T) + 1e-30
    ratio = np.abs(y - ref) / bound
    assert ratio.max() <= 1.0, f"worst error {ratio.max():.3f} x the bound"
    return ratio.max()


@pytest.mark.parametrize("d_out,d_in,g,m", [(32, 128, -1, 1), (100, 640, 128, 3), (4096, 4096, 128, 1),
                                            (4096, 4096, 128, 8), (300, 1024, -1, 8), (1000, 2048, 256, 5),
                                            (7, 384, 128, 2)])
def test_gemv_matches_oracle(d_out, d_in, g, m):
    words, s, z = _stored_form(d_out, d_in, g, d_out + d_in)
    xbits, xf = _tokens(m, d_in, d_in)
    y = _run(words, s, z, g, xbits)
    _check(y, words, s, z, g, xf)


@pytest.mark.parametrize("d_out,d_in,g,m", [(4096, 4096, 128, 4), (50, 384, -1, 2)])
def test_gemv_act_order_permutation(d_out, d_in, g, m):
    words, s, z = _stored_form(d_out, d_in, g, 7 * d_out + d_in)
    xbits, xf = _tokens(m, d_in, 3)
    perm = np.random.default_rng(d_in).permutation(d_in)
    y = _run(words, s, z, g, xbits, perm)
    _check(y, words, s, z, g, xf, perm)


@pytest.mark.parametrize("g,m,with_perm", [(128, 8, False), (128, 8, True), (-1, 1, False)])
def test_gemv_widest_rows(g, m, with_perm):
    """d_in = 32768, the widest the library takes: the most column blocks,
    the largest staged scale table (256 groups) and, at m = 8, the largest
    block data of x (the ring drops to two stages); 70 rows, a ragged tile."""
    d_out, d_in = 70, 32768
    words, s, z = _stored_form(d_out, d_in, g, 11 + m)
    xbits, xf = _tokens(m, d_in, 13)
    perm = np.random.default_rng(4).permutation(d_in) if with_perm else None
    y = _run(words, s, z, g, xbits, perm)
    _check(y, words, s, z, g, xf, perm)


@pytest.mark.parametrize("m", [1, 8])
def test_gemv_full_size_sampled_rows(m):
    """The 8192 x 28672 g128 layer (the largest of the workloads), every
    output computed; 64 rows checked against the oracle, first and last
    included."""
    d_out, d_in, g = 8192, 28672, 128
    words, s, z = _stored_form(d_out, d_in, g, 5)
    xbits, xf = _tokens(m, d_in, 9)
    y = _run(words, s, z, g, xbits)
    assert np.isfinite(y).all()
    rows = np.unique(np.concatenate([[0, d_out - 1], np.random.default_rng(1).choice(d_out, 62, replace=False)]))
    _check(y, words, s, z, g, xf, rows=rows)


def test_gemv_of_a_quantized_layer():
    """The GPU's own act-order quantization of a d_model=768 GPT layer, then
    the product from its stored form against x Q^T from its Q."""
    p = dataclasses.replace(synth.gpt768_layer(1, rows_per_batch=1024, n_batches=2), groupsize=128)
    xs = [to_dev_x(p, p.x_batch(b)) for b in range(p.n_batches)]
    lq = api.LayerQuantizer(p.d_out, p.d_in, 4, 128, 128, p.percdamp, want_q=True, act_order=True)
    lq.begin(torch.from_numpy(p.W).cuda())
    lq.add_batches(xs)
    lq.finish()
    api.get_status()
    xbits, xf = _tokens(6, p.d_in, 11)
    xd = torch.from_numpy(xbits.view(np.int16)).cuda().view(torch.bfloat16)
    y = torch.empty((6, p.d_out), dtype=torch.float32, device="cuda")
    api.dequant_gemv(lq.codes, lq.scales, lq.zeros, 4, 128, xd, y, perm=lq.perm)
    api.get_status()
    Q = lq.Q.cpu().numpy().astype(np.float64)
    ref = xf.astype(np.float64) @ Q.T
    bound = TOL * (np.abs(xf.astype(np.float64)) @ np.abs(Q).T)
    assert (np.abs(y.cpu().numpy() - ref) <= bound).all()
    # and the oracle, from the same stored form
    words = lq.codes.cpu().numpy().view(np.uint32)
    s, z = lq.scales.cpu().numpy(), lq.zeros.cpu().numpy()
    _check(y.cpu().numpy().astype(np.float64), words, s, z, 128, xf, lq.perm.cpu().numpy())


def test_gemv_bad_permutation_entry_is_reported():
    d_out, d_in = 64, 256
    words, s, z = _stored_form(d_out, d_in, 128, 1)
    xbits, _ = _tokens(2, d_in, 2)
    codes, sd, zd, xd = _dev(words, s, z, xbits)
    perm = torch.arange(d_in, dtype=torch.int32, device="cuda")
    perm[17] = d_in + 5                    # checked before use: never an address
    y = torch.zeros((2, d_out), dtype=torch.float32, device="cuda")
    api.dequant_gemv(codes, sd, zd, 4, 128, xd, y, perm=perm)
    with pytest.raises(api.GPTQError) as e:
        api.get_status()
    assert e.value.code == 1
    assert torch.isnan(y).all()


def test_gemv_no_tokens_and_unsupported_widths():
    words, s, z = _stored_form(32, 128, -1, 1)
    codes, sd, zd, _ = _dev(words, s, z, np.zeros((1, 128), np.uint16))
    y = torch.full((0, 32), 1.0, dtype=torch.float32, device="cuda")
    x0 = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    api.dequant_gemv(codes, sd, zd, 4, -1, x0, y)          # m = 0: nothing to do
    x1 = torch.zeros((1, 128), dtype=torch.bfloat16, device="cuda")
    y1 = torch.empty((1, 32), dtype=torch.float32, device="cuda")
    c3 = torch.zeros((32, 128 * 3 // 32), dtype=torch.int32, device="cuda")
    with pytest.raises(api.GPTQError) as e:
        api.dequant_gemv(c3, sd, zd, 3, -1, x1, y1)
    assert e.value.code == 2
