"""GPU parity of gptq_dequantize (note "Model Quantization", "주요 양자화 기법":
the INT4 weights restored to FP16 for the computation; blog section 5): the
weights rebuilt from the stored form, bit-exact against the oracle's
s (c - z) in fp32, and against its round-to-nearest-even in bf16 / fp16."""
import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_05_b200 import api, build_lib, synth
from parity_util import to_dev_x

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _ready():
    build_lib.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    api.get_status(raise_on_error=False)
    yield
    code, _ = api.get_status(raise_on_error=False)
    assert code == 0


def _stored(d_out, d_in, bits, g, seed):
    rng = np.random.default_rng(seed)
    words = rng.integers(0, 2 ** 32, size=(d_out, d_in * bits // 32), dtype=np.uint64).astype(np.uint32)
    ng = 1 if g <= 0 else d_in // g
    s = (np.abs(rng.standard_normal((d_out, ng))) * 3e-3 + 1e-4).astype(np.float16)
    z = rng.integers(0, 2 ** bits, size=(d_out, ng)).astype(np.float16)
    z[::5, 0] = -3.0
    return words, s, z


def _expected(words, s, z, bits, g, d_in, perm):
    c = oracle.unpack_codes(words, bits, d_in)
    gi = np.arange(d_in) // (d_in if g <= 0 else g)
    Qp = oracle.dequant(c, s.astype(np.float64)[:, gi], z.astype(np.float64)[:, gi])   # processing order, exact
    if perm is None:
        return Qp
    Q = np.full_like(Qp, np.nan)
    Q[:, perm] = Qp
    return Q


def _run(words, s, z, bits, g, d_in, perm, dtype):
    out = torch.empty((words.shape[0], d_in), dtype=dtype, device="cuda")
    pd = None if perm is None else torch.from_numpy(np.asarray(perm, dtype=np.int32)).cuda()
    api.dequantize(torch.from_numpy(words.view(np.int32)).cuda(), torch.from_numpy(s).cuda(),
                   torch.from_numpy(z).cuda(), bits, g, out, perm=pd)
    api.get_status()
    return out


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("g,with_perm", [(-1, False), (128, False), (128, True), (256, True)])
def test_dequantize_bit_exact(bits, g, with_perm):
    d_out, d_in = 300, 1024
    words, s, z = _stored(d_out, d_in, bits, g, bits * 10 + (g > 0) + 2 * with_perm)
    perm = np.random.default_rng(bits).permutation(d_in) if with_perm else None
    want = _expected(words, s, z, bits, g, d_in, perm)
    got = _run(words, s, z, bits, g, d_in, perm, torch.float32).cpu().numpy()
    assert np.array_equal(got.astype(np.float64), want)        # fp32 is exact
    for dt in (torch.bfloat16, torch.float16):
        got = _run(words, s, z, bits, g, d_in, perm, dt).cpu()
        assert torch.equal(got, torch.from_numpy(want.astype(np.float32)).to(dt))


def test_dequantize_equals_the_quantizers_q():
    """The stored form of a GPU act-order quantization rebuilds exactly the Q
    the sweep wrote."""
    import dataclasses
    p = dataclasses.replace(synth.gpt768_layer(1, rows_per_batch=1024, n_batches=2), groupsize=128)
    lq = api.LayerQuantizer(p.d_out, p.d_in, 4, 128, 128, p.percdamp, want_q=True, act_order=True)
    lq.begin(torch.from_numpy(p.W).cuda())
    lq.add_batches([to_dev_x(p, p.x_batch(b)) for b in range(p.n_batches)])
    lq.finish()
    out = torch.empty((p.d_out, p.d_in), dtype=torch.float32, device="cuda")
    api.dequantize(lq.codes, lq.scales, lq.zeros, 4, 128, out, perm=lq.perm)
    api.get_status()
    assert torch.equal(out, lq.Q)


@pytest.mark.parametrize("bits", [3, 4])
def test_dequantize_full_size_sampled_rows(bits):
    d_out, d_in, g = 8192, 28672, 128
    words, s, z = _stored(d_out, d_in, bits, g, 99)
    perm = np.random.default_rng(5).permutation(d_in)
    out = _run(words, s, z, bits, g, d_in, perm, torch.bfloat16)
    rows = np.unique(np.concatenate([[0, d_out - 1], np.random.default_rng(6).choice(d_out, 30, replace=False)]))
    want = _expected(words[rows], s[rows], z[rows], bits, g, d_in, perm)
    assert torch.equal(out[torch.from_numpy(rows).cuda()].cpu(), torch.from_numpy(want.astype(np.float32)).bfloat16())


def test_dequantize_bad_permutation_entry_is_reported():
    d_in = 256
    words, s, z = _stored(8, d_in, 4, -1, 1)
    perm = np.arange(d_in)
    perm[3] = -7
    with pytest.raises(api.GPTQError):
        _run(words, s, z, 4, -1, d_in, perm, torch.float32)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("d_out,d_in,g", [(1, 128, -1), (7, 384, 128), (3, 32768, 256)])
def test_dequantize_edge_shapes(bits, d_out, d_in, g):
    """One row of the narrowest width, a ragged row count, and the widest rows
    (the permuted path's largest shared-memory footprint), with and without a
    permutation."""
    words, s, z = _stored(d_out, d_in, bits, g, d_out * 100 + bits)
    for with_perm in (False, True):
        perm = np.random.default_rng(d_in + bits).permutation(d_in) if with_perm else None
        want = _expected(words, s, z, bits, g, d_in, perm)
        got = _run(words, s, z, bits, g, d_in, perm, torch.float32).cpu().numpy()
        assert np.array_equal(got.astype(np.float64), want)
        got = _run(words, s, z, bits, g, d_in, perm, torch.bfloat16).cpu()
        assert torch.equal(got, torch.from_numpy(want.astype(np.float32)).bfloat16())


@pytest.mark.parametrize("with_perm", [False, True])
def test_dequantize_rounds_once(with_perm):
    """Zero points off the integers (any fp16 grid a caller brings): each value
    is the exact s (c - z) rounded once to fp32, then to nearest even for
    fp16 / bf16.  The products here need up to 25 significant bits, so fp32
    rounding does occur."""
    d_out, d_in, g = 64, 1024, 128
    words, s, z = _stored(d_out, d_in, 4, g, 17)
    rng = np.random.default_rng(18)
    z = rng.uniform(-8.0, 24.0, size=z.shape).astype(np.float16)
    perm = np.random.default_rng(19).permutation(d_in) if with_perm else None
    want = _expected(words, s, z, 4, g, d_in, perm)           # exact in fp64
    want32 = want.astype(np.float32)
    assert np.any(want32.astype(np.float64) != want)            # some values do round
    got = _run(words, s, z, 4, g, d_in, perm, torch.float32).cpu().numpy()
    assert np.array_equal(got, want32)
    for dt in (torch.bfloat16, torch.float16):
        got = _run(words, s, z, 4, g, d_in, perm, dt).cpu()
        assert torch.equal(got, torch.from_numpy(want32).to(dt))
