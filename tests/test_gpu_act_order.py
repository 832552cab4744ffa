"""GPU parity of act-order (itwiki "GPTQ", "실무 변형"): the processing order,
the permuted Hessian and the column permutations bit-exact against the
oracle / numpy indexing, and the whole act-order layer against
oracle.gptq_quantize_act_order."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_05_b200 import api, build_lib, synth
from parity_util import (H_TOL, LOSS_TOL, check_codes, dequant_rows, fp16_values, rel_fro, to_dev_x,
                         unpack_gpu_codes, upper)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _ready():
    build_lib.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    api.get_status(raise_on_error=False)
    yield
    code, _ = api.get_status(raise_on_error=False)
    assert code == 0


def _diag_with_ties(d, seed):
    """A diagonal with repeated values, both zeros, negatives, infinities and
    NaNs (the order must be total and stable on all of them)."""
    rng = np.random.default_rng(seed)
    v = rng.lognormal(0.0, 1.0, size=d).astype(np.float32)
    idx = rng.permutation(d)
    v[idx[: d // 8]] = v[idx[d // 8: d // 4]]          # many exact ties
    v[idx[d // 4]] = 0.0
    v[idx[d // 4 + 1]] = -0.0
    v[idx[d // 4 + 2]] = 0.0
    v[idx[d // 4 + 3]] = -1.5
    v[idx[d // 4 + 4]] = np.inf
    v[idx[d // 4 + 5]] = -np.inf
    v[idx[d // 4 + 6]] = np.nan
    v[idx[d // 4 + 7]] = np.nan
    return v


@pytest.mark.parametrize("d", [128, 640, 4096, 32768])
def test_act_order_perm_bit_exact(d):
    diag = _diag_with_ties(d, d)
    H = torch.empty((d, d), dtype=torch.float32, device="cuda")     # only the diagonal is read
    H.view(-1)[:: d + 1] = torch.from_numpy(diag).cuda()
    perm = torch.full((d,), -1, dtype=torch.int32, device="cuda")
    api.act_order_perm(H, perm)
    api.get_status()
    want = np.argsort(-diag.astype(np.float64), kind="stable")
    # the oracle sorts a diagonal matrix's diagonal the same way
    if d <= 640:
        assert np.array_equal(want, oracle.act_order_perm(np.diag(diag.astype(np.float64))))
    assert np.array_equal(perm.cpu().numpy(), want)


def test_act_order_perm_of_sorted_and_constant_diagonals():
    d = 384
    for diag in (np.linspace(5.0, 1.0, d), np.linspace(1.0, 5.0, d), np.full(d, 2.0)):
        H = torch.from_numpy(np.diag(diag).astype(np.float32)).cuda()
        perm = torch.empty((d,), dtype=torch.int32, device="cuda")
        api.act_order_perm(H, perm)
        api.get_status()
        assert np.array_equal(perm.cpu().numpy(), oracle.act_order_perm(np.diag(diag)))


def _sym_upper_with_garbage_below(d, seed):
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((d, d)).astype(np.float32)
    S = np.triu(A) + np.triu(A, 1).T
    Hg = np.triu(A).copy()
    Hg[np.tril_indices(d, -1)] = np.nan         # must never be read
    return S, Hg


@pytest.mark.parametrize("d", [128, 640, 4096])
def test_permute_hessian_bit_exact(d):
    S, Hg = _sym_upper_with_garbage_below(d, d + 1)
    rng = np.random.default_rng(d)
    p = rng.permutation(d).astype(np.int32)
    H = torch.from_numpy(Hg).cuda()
    Hp = torch.full((d, d), 7.0, dtype=torch.float32, device="cuda")
    api.permute_hessian(H, torch.from_numpy(p).cuda(), Hp)
    api.get_status()
    assert np.array_equal(Hp.cpu().numpy(), S[np.ix_(p, p)])


@pytest.mark.parametrize("rows,cols", [(1, 128), (300, 640), (4096, 4096), (3, 32768)])
@pytest.mark.parametrize("in_place", [False, True])
def test_permute_columns_bit_exact(rows, cols, in_place):
    rng = np.random.default_rng(rows * 7 + cols)
    A = rng.standard_normal((rows, cols)).astype(np.float32)
    p = rng.permutation(cols).astype(np.int32)
    pt = torch.from_numpy(p).cuda()
    src = torch.from_numpy(A).cuda()
    dst = src if in_place else torch.empty_like(src)
    api.permute_columns(src, pt, dst)
    api.get_status()
    fwd = A[:, p]
    assert np.array_equal(dst.cpu().numpy(), fwd)
    back = dst if in_place else torch.empty_like(src)
    api.permute_columns(dst, pt, back, inverse=True)
    api.get_status()
    assert np.array_equal(back.cpu().numpy(), A)


def test_bad_permutation_entry_is_reported_not_read():
    d = 256
    p = np.arange(d, dtype=np.int32)[::-1].copy()
    p[5] = d + 1000                  # outside [0, d): checked before any use as an index
    p[9] = -3
    pt = torch.from_numpy(p).cuda()
    A = torch.ones((4, d), dtype=torch.float32, device="cuda")
    out = torch.empty_like(A)
    api.permute_columns(A, pt, out)
    with pytest.raises(api.GPTQError) as e:
        api.get_status()
    assert e.value.code == 1
    o = out.cpu().numpy()
    assert np.isnan(o[:, [5, 9]]).all() and (np.delete(o, [5, 9], axis=1) == 1.0).all()
    H = torch.eye(d, dtype=torch.float32, device="cuda")
    Hp = torch.empty_like(H)
    api.permute_hessian(H, pt, Hp)
    with pytest.raises(api.GPTQError):
        api.get_status()
    h = Hp.cpu().numpy()
    assert np.isnan(h[[5, 9], :]).all() and np.isnan(h[:, [5, 9]]).all()


def _act_order_layer(p, xs_dev, want_q=True):
    lq = api.LayerQuantizer(p.d_out, p.d_in, p.bits, p.groupsize, 128, p.percdamp, want_q=want_q, act_order=True)
    lq.begin(torch.from_numpy(p.W).cuda())
    lq.add_batches(xs_dev)
    lq.finish()
    api.get_status()
    return lq


@pytest.mark.parametrize("layer,bits,g", [(1, 4, -1), (1, 4, 128), (2, 3, -1), (3, 4, 256)])
def test_act_order_layer_end_to_end(layer, bits, g):
    """gpt768 layers (per-channel std LogNormal(0, 0.5): uneven input energy)
    with act-order against the oracle's act-order GPTQ."""
    p = dataclasses.replace(synth.gpt768_layer(layer, rows_per_batch=1024, n_batches=3), bits=bits, groupsize=g)
    xs = [p.x_batch(b) for b in range(p.n_batches)]
    lq = _act_order_layer(p, [to_dev_x(p, x) for x in xs])
    H = oracle.hessian([synth.x_as_f32(p, x) for x in xs])
    Hg = lq.H.cpu().numpy()
    assert rel_fro(upper(Hg), upper(H)) <= H_TOL
    # the order is decided on the fp32 diagonal on both sides
    perm = lq.perm.cpu().numpy()
    assert np.array_equal(perm, oracle.act_order_perm(np.diag(np.diag(Hg).astype(np.float64))))
    assert np.array_equal(lq.Hp.cpu().numpy(), (np.triu(Hg) + np.triu(Hg, 1).T)[np.ix_(perm, perm)])
    ref = oracle.gptq_quantize_act_order(p.W, H, bits, 128, g, p.percdamp, perm=perm, return_trace=True)
    got = unpack_gpu_codes(lq.codes, bits, p.d_in)
    s, z = fp16_values(lq.scales), fp16_values(lq.zeros)
    check_codes(got, ref, "act-order", groupsize=g, gpu_scales=s, gpu_zeros=z)
    Qg = lq.Q.cpu().numpy().astype(np.float64)
    # Q is in W's column order and lies on the recorded grid of the processing order
    assert np.array_equal(Qg[:, perm], dequant_rows(got, s, z, g))
    lg = oracle.layer_loss_hessian(p.W, Qg, H)
    lo = oracle.layer_loss_hessian(p.W, ref["Q"], H)
    assert abs(lg / lo - 1.0) <= LOSS_TOL


def test_act_order_beats_natural_order_on_outlier_channels():
    """On inputs with a few x20 channels (the Llama MLP recipe, reduced in
    size) act-order gives a lower layer loss than the natural order."""
    d_out, d_in, n = 512, 1024, 8192
    rng = synth.rng_for("smoke", 77, 0, 3)
    scale = np.ones(d_in, np.float32)
    scale[rng.choice(d_in, size=d_in // 100, replace=False)] = 20.0
    W = synth.round_to_bf16(synth.normal_weights(synth.rng_for("smoke", 77, 0, 0), d_out, d_in, 0.02))

    def xf(b):
        x = synth.ar1_rows(synth.rng_for("smoke", 77, b, 1), n // 2, d_in, 0.5, "t3") * scale[None, :]
        return synth.f32_to_bf16_bits(x)

    p = synth.LayerProblem("outlier", d_out, d_in, 4, -1, 128, 0.01, "bf16", "bf16", 2, n // 2, W, _x_fn=xf)
    xs = [p.x_batch(b) for b in range(2)]
    xs_dev = [to_dev_x(p, x) for x in xs]
    act = _act_order_layer(p, xs_dev)
    nat = api.LayerQuantizer(d_out, d_in, 4, -1, 128, 0.01, want_q=True)
    nat.begin(torch.from_numpy(W).cuda())
    nat.add_batches(xs_dev)
    nat.finish()
    api.get_status()
    H = oracle.hessian([synth.x_as_f32(p, x) for x in xs])
    la = oracle.layer_loss_hessian(W, act.Q.cpu().numpy().astype(np.float64), H)
    ln = oracle.layer_loss_hessian(W, nat.Q.cpu().numpy().astype(np.float64), H)
    assert la < ln
