"""Seeded synthetic inputs for the GPTQ layer quantizer.

This module is shared by the CUDA path (bench, tests) and the fp64 oracle
(tests only).  It holds none of the method's arithmetic: it only draws random
weights W and calibration activations X with the shapes and statistics of the
workloads below, and converts fp32 to bf16 bit patterns.

Workloads (all weights random-init, all activations synthetic; no dataset or
checkpoint is used):

* ``smoke``      W [512, 512] fp32 ~ N(0, 0.02^2); X [2048, 512] fp32 with an
                 AR(1) channel correlation rho = 0.9 (the correlated 512-dim,
                 2048-sample example of the itwiki "GPTQ" article, section
                 "최소 구현").
* ``gpt768``     the 48 linear layers of a 12-block GPT with d_model = 768;
                 per layer 20480 bf16 calibration rows in 10 batches, AR(1)
                 rho = 0.8, per-channel std ~ LogNormal(0, 0.5).
* ``attn4096``   W [4096, 4096] bf16 ~ N(0, 0.02^2); X 262144 x 4096 bf16,
                 AR(1) rho = 0.9, 16 batches of 16384 rows.
* ``mlp11008``   up [11008, 4096] / down [4096, 11008] bf16 ~ N(0, 0.02^2);
                 65536 rows of Student-t(3) innovations, AR(1) rho = 0.5, 1% of
                 channels (seed-chosen) scaled x20.
* ``mlp28672``   W [8192, 28672] bf16 ~ N(0, 0.01^2); X 65536 x 28672 bf16,
                 AR(1) rho = 0.9, 8 batches of 8192 rows.
* ``gptstack``   weights of a stack of pre-LN GPT blocks (qkv [3d, d],
                 attn_out [d, d], fc [4d, d], mlp_proj [d, 4d], all ~ N(0, 0.02^2),
                 no biases, LayerNorms with unit gain and zero shift) and the
                 calibration activations fed to its first block: batches of
                 [seqs, tokens, d] with the gpt768 channel statistics (AR(1)
                 rho = 0.8, per-channel std LogNormal(0, 0.5)).  Whole-model
                 calibration passes them through the blocks in order.

The AR(1) rows are drawn by the exact recursion x_0 = z_0,
x_a = rho * x_{a-1} + sqrt(1 - rho^2) * z_a over the channel index a, which
has covariance Sigma_ab = rho^|a-b| (the same law as Z C^T with C the
Cholesky factor of Sigma) at O(n d) cost.

Every array is a pure function of (workload, layer, batch, base seed): the
generator is ``numpy.random.default_rng([base_seed, workload_id, layer, batch,
stream])`` (PCG64 seeded through a SeedSequence).
"""
from __future__ import annotations

import dataclasses
import numpy as np

WORKLOAD_IDS = {"smoke": 1, "gpt768": 2, "attn4096": 3, "mlp11008": 4, "mlp28672": 5, "gptstack": 6}

_STREAM_W = 0
_STREAM_X = 1
_STREAM_SCALE = 2
_STREAM_OUTLIER = 3


def rng_for(workload: str, layer: int, batch: int, stream: int, base_seed: int = 0):
    """PCG64 generator for one (workload, layer, batch, stream) tuple."""
    return np.random.default_rng([base_seed, WORKLOAD_IDS[workload], layer, batch, stream])


# ---------------------------------------------------------------------------
# bf16 bit patterns (round to nearest even), kept here so that both sides see
# the very same bytes.
# ---------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit pattern (uint16), round-to-nearest-even.  Inputs are
    finite (the generators never produce NaN/Inf)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit pattern (uint16) -> fp32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 values rounded to the nearest bf16 value, returned as fp32."""
    return bf16_bits_to_f32(f32_to_bf16_bits(x))


# ---------------------------------------------------------------------------
# Primitive draws
# ---------------------------------------------------------------------------
def ar1_rows(rng, n: int, d: int, rho: float, innovations: str = "normal",
             chunk: int = 1 << 14) -> np.ndarray:
    """[n, d] fp32 rows with AR(1) correlation rho along the channel axis.

    ``innovations`` is ``"normal"`` (N(0,1)) or ``"t3"`` (Student-t, nu = 3).
    Innovations are drawn channel-major per chunk of rows (shape
    [d, rows]) so that the recursion runs over contiguous vectors."""
    out = np.empty((n, d), dtype=np.float32)
    c = np.float32(np.sqrt(1.0 - rho * rho))
    r = np.float32(rho)
    for r0 in range(0, n, chunk):
        r1 = min(n, r0 + chunk)
        if innovations == "normal":
            z = rng.standard_normal((d, r1 - r0), dtype=np.float32)
        elif innovations == "t3":
            z = rng.standard_t(3.0, size=(d, r1 - r0)).astype(np.float32)
        else:
            raise ValueError(innovations)
        for a in range(1, d):
            z[a] *= c
            z[a] += r * z[a - 1]
        for a0 in range(0, d, 64):          # tiled transpose back to row-major
            for s0 in range(0, r1 - r0, 1024):
                s1 = min(r1 - r0, s0 + 1024)
                out[r0 + s0:r0 + s1, a0:a0 + 64] = z[a0:a0 + 64, s0:s1].T
    return out


def normal_weights(rng, d_out: int, d_in: int, std: float) -> np.ndarray:
    return (rng.standard_normal((d_out, d_in), dtype=np.float32) * np.float32(std))


# ---------------------------------------------------------------------------
# Workloads
# ---------------------------------------------------------------------------
@dataclasses.dataclass
class LayerProblem:
    """One layer to quantize.

    W        fp32 [d_out, d_in] (bf16-representable when ``w_dtype == 'bf16'``)
    x_dtype  'f32' or 'bf16'; X batches are fp32 arrays for 'f32' and uint16
             bf16 bit patterns for 'bf16'
    """
    name: str
    d_out: int
    d_in: int
    bits: int
    groupsize: int
    blocksize: int
    percdamp: float
    w_dtype: str
    x_dtype: str
    n_batches: int
    batch_rows: int
    W: np.ndarray
    last_batch_rows: int = 0
    _x_fn: object = dataclasses.field(repr=False, default=None)

    def x_batch(self, b: int) -> np.ndarray:
        return self._x_fn(b)

    def x_batches(self):
        for b in range(self.n_batches):
            yield self.x_batch(b)

    def rows_in_batch(self, b: int) -> int:
        if b == self.n_batches - 1 and self.last_batch_rows:
            return self.last_batch_rows
        return self.batch_rows

    @property
    def n(self) -> int:
        return sum(self.rows_in_batch(b) for b in range(self.n_batches))


def smoke(base_seed: int = 0) -> LayerProblem:
    """W [512,512] fp32, X [2048,512] fp32 AR(1) rho=0.9; 4-bit per-row."""
    W = normal_weights(rng_for("smoke", 0, 0, _STREAM_W, base_seed), 512, 512, 0.02)

    def xf(b):
        return ar1_rows(rng_for("smoke", 0, b, _STREAM_X, base_seed), 2048, 512, 0.9)

    return LayerProblem("smoke", 512, 512, 4, -1, 128, 0.01, "f32", "f32", 1, 2048, W, _x_fn=xf)


GPT768_SHAPES = (("qkv", 2304, 768), ("attn_out", 768, 768), ("fc", 3072, 768), ("mlp_proj", 768, 3072))


def gpt768_layer(layer: int, base_seed: int = 0, rows_per_batch: int = 2048,
                 n_batches: int = 10) -> LayerProblem:
    """Layer ``layer`` (0..47) of the 12-block d_model=768 GPT: block layer//4,
    kind GPT768_SHAPES[layer % 4]; 10 batches x 8 seqs x 256 tokens of bf16
    activations, AR(1) rho = 0.8, per-channel std LogNormal(0, 0.5)."""
    kind, d_out, d_in = GPT768_SHAPES[layer % 4]
    W = normal_weights(rng_for("gpt768", layer, 0, _STREAM_W, base_seed), d_out, d_in, 0.02)
    ch_scale = np.exp(rng_for("gpt768", layer, 0, _STREAM_SCALE, base_seed)
                      .normal(0.0, 0.5, size=d_in)).astype(np.float32)

    def xf(b):
        x = ar1_rows(rng_for("gpt768", layer, b, _STREAM_X, base_seed), rows_per_batch, d_in, 0.8)
        x *= ch_scale[None, :]
        return f32_to_bf16_bits(x)

    return LayerProblem(f"gpt768.{layer // 4}.{kind}", d_out, d_in, 4, -1, 128, 0.01, "f32",
                        "bf16", n_batches, rows_per_batch, W, _x_fn=xf)


def attn4096(base_seed: int = 0, n_batches: int = 16, batch_rows: int = 16384) -> LayerProblem:
    """W [4096,4096] bf16; X 16 x 16384 rows bf16, AR(1) rho = 0.9; 4-bit g=128."""
    W = round_to_bf16(normal_weights(rng_for("attn4096", 0, 0, _STREAM_W, base_seed), 4096, 4096, 0.02))

    def xf(b):
        return f32_to_bf16_bits(ar1_rows(rng_for("attn4096", 0, b, _STREAM_X, base_seed), batch_rows, 4096, 0.9))

    return LayerProblem("attn4096", 4096, 4096, 4, 128, 128, 0.01, "bf16", "bf16", n_batches,
                        batch_rows, W, _x_fn=xf)


def mlp11008(which: str, bits: int, base_seed: int = 0, n_batches: int = 8,
             batch_rows: int = 8192) -> LayerProblem:
    """Llama-7B MLP pair: which = 'up' ([11008, 4096]) or 'down' ([4096, 11008]);
    65536 rows of Student-t(3) innovations with AR(1) rho = 0.5, and
    round(0.01 * d_in) seed-chosen channels scaled x20.  Per-row grid."""
    layer = 0 if which == "up" else 1
    d_out, d_in = (11008, 4096) if which == "up" else (4096, 11008)
    W = round_to_bf16(normal_weights(rng_for("mlp11008", layer, 0, _STREAM_W, base_seed), d_out, d_in, 0.02))
    n_out = int(round(0.01 * d_in))
    outliers = rng_for("mlp11008", layer, 0, _STREAM_OUTLIER, base_seed).choice(d_in, size=n_out, replace=False)
    scale = np.ones(d_in, dtype=np.float32)
    scale[outliers] = 20.0

    def xf(b):
        x = ar1_rows(rng_for("mlp11008", layer, b, _STREAM_X, base_seed), batch_rows, d_in, 0.5, "t3")
        x *= scale[None, :]
        return f32_to_bf16_bits(x)

    return LayerProblem(f"mlp11008.{which}.int{bits}", d_out, d_in, bits, -1, 128, 0.01, "bf16",
                        "bf16", n_batches, batch_rows, W, _x_fn=xf)


def mlp28672(base_seed: int = 0, n_batches: int = 8, batch_rows: int = 8192) -> LayerProblem:
    """W [8192, 28672] bf16 ~ N(0, 0.01^2); X 8 x 8192 rows bf16 AR(1) 0.9; 4-bit g=128."""
    W = round_to_bf16(normal_weights(rng_for("mlp28672", 0, 0, _STREAM_W, base_seed), 8192, 28672, 0.01))

    def xf(b):
        return f32_to_bf16_bits(ar1_rows(rng_for("mlp28672", 0, b, _STREAM_X, base_seed), batch_rows, 28672, 0.9))

    return LayerProblem("mlp28672", 8192, 28672, 4, 128, 128, 0.01, "bf16", "bf16", n_batches,
                        batch_rows, W, _x_fn=xf)


def custom(name: str, d_out: int, d_in: int, n: int, *, bits: int = 4, groupsize: int = -1,
           rho: float = 0.9, x_dtype: str = "bf16", innovations: str = "normal",
           w_std: float = 0.02, n_batches: int = 1, base_seed: int = 0, layer: int = 0) -> LayerProblem:
    """A small problem with the same statistics, for parity tests at sizes the
    oracle finishes in seconds (ragged row counts, odd block counts...)."""
    rows = -(-n // n_batches)
    W = normal_weights(rng_for("smoke", 1000 + layer, 0, _STREAM_W, base_seed), d_out, d_in, w_std)
    if x_dtype == "bf16":
        W = round_to_bf16(W)

    def xf(b):
        r = min(rows, n - b * rows)
        x = ar1_rows(rng_for("smoke", 1000 + layer, b, _STREAM_X, base_seed), r, d_in, rho, innovations)
        return f32_to_bf16_bits(x) if x_dtype == "bf16" else x

    return LayerProblem(name, d_out, d_in, bits, groupsize, 128, 0.01,
                        "bf16" if x_dtype == "bf16" else "f32", x_dtype, n_batches, rows, W,
                        n - (n_batches - 1) * rows, _x_fn=xf)


def x_batches_threaded(problem: LayerProblem, workers: int = 8):
    """All calibration batches of ``problem``, drawn concurrently in threads
    (each batch has its own generator, so the result does not depend on the
    thread count)."""
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=max(1, workers)) as ex:
        return list(ex.map(problem.x_batch, range(problem.n_batches)))


def x_as_f32(problem: LayerProblem, xb: np.ndarray) -> np.ndarray:
    """A batch as fp32 values (exact widening of the bf16 bytes)."""
    return bf16_bits_to_f32(xb) if problem.x_dtype == "bf16" else np.asarray(xb, dtype=np.float32)


# ---------------------------------------------------------------------------
# A stack of GPT blocks for block-sequential calibration
# ---------------------------------------------------------------------------
GPT_LINEARS = ("qkv", "attn_out", "fc", "mlp_proj")


def gpt_stack_weights(n_blocks: int, d_model: int, base_seed: int = 0, w_std: float = 0.02):
    """Per block a dict name -> fp32 weight [d_out, d_in] (nn.Linear layout)."""
    shapes = {"qkv": (3 * d_model, d_model), "attn_out": (d_model, d_model), "fc": (4 * d_model, d_model),
              "mlp_proj": (d_model, 4 * d_model)}
    blocks = []
    for b in range(n_blocks):
        blocks.append({name: normal_weights(rng_for("gptstack", b, i, _STREAM_W, base_seed), *shapes[name], w_std)
                       for i, name in enumerate(GPT_LINEARS)})
    return blocks


def gpt_stack_inputs(n_batches: int, seqs: int, tokens: int, d_model: int, base_seed: int = 0):
    """Calibration activations entering the first block: n_batches arrays
    [seqs, tokens, d_model] fp32 (AR(1) rho = 0.8 over channels, per-channel
    std LogNormal(0, 0.5))."""
    ch_scale = np.exp(rng_for("gptstack", 0, 0, _STREAM_SCALE, base_seed).normal(0.0, 0.5, size=d_model))
    out = []
    for b in range(n_batches):
        x = ar1_rows(rng_for("gptstack", 0, b, _STREAM_X, base_seed), seqs * tokens, d_model, 0.8)
        out.append((x * ch_scale[None, :].astype(np.float32)).reshape(seqs, tokens, d_model))
    return out
