"""Seeded synthetic workloads for the W4A16 quantized linear layer.

This module is the only code shared by the tests, the benchmark, the oracle and the
product binding.  It draws random inputs with the shapes and value distributions of the
pages' workloads (Llama-family linear layers) and holds none of the method's arithmetic:
no scale formula, no quantizer, no product, no outlier selection.

Distributions (the pages' models and calibration sets are not available, so these
stand in for them):
  W            fp32 [N][K] ~ N(0, 0.02^2)
  m_k          lognormal(0, 1) per input channel; 8 distinct channels drawn uniformly
               and multiplied by 20 (activation outlier channels)
  act_absmean  mean over a calibration batch X_cal[512][K] = N(0,1) * m_k of |X_cal|,
               summed in fp64, stored fp32
  x'           bf16 [M][K] = bf16_rne(N(0,1) * m_k^(1 - alpha)): the runtime activation
               after the caller has folded 1/s into the previous operator, drawn directly
               with the per-channel spread that x / s has when s ~ m_k^alpha

Seeds: seed = 1000 * config + shape_index, with independent substreams (numpy PCG64
SeedSequence.spawn) for W, the multipliers, the outlier channels, the calibration batch
and x.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

# (K, N) shapes of the pages' model families: out x in weights W[N][K].
LLAMA3_8B = [("qkv_proj", 4096, 6144), ("o_proj", 4096, 4096), ("gate_up_proj", 4096, 28672),
             ("down_proj", 14336, 4096)]
LLAMA2_13B = [("attn_5120x5120", 5120, 5120), ("mlp_5120x13824", 5120, 13824)]
LLAMA2_70B = [("qkv_proj", 8192, 10240), ("o_proj", 8192, 8192), ("gate_up_proj", 8192, 57344),
              ("down_proj", 28672, 8192)]

# Workloads (M = tokens).  `family` numbers the seeds of a workload's layers (seed_of).
SINGLE_LAYER = dict(family=0, name="single layer 4096x4096, M=1", shapes=[("layer", 4096, 4096)], Ms=[1],
                    csr=False)
DECODE_SWEEP = dict(family=1, name="decode GEMV sweep, Llama-3-8B shapes", shapes=LLAMA3_8B, Ms=[1, 4, 8, 16],
                    csr=False)
PREFILL_SWEEP = dict(family=2, name="prefill GEMM, Llama-3-8B shapes", shapes=LLAMA3_8B, Ms=[512, 2048, 8192],
                     csr=False)
DENSE_SPARSE_13B = dict(family=3, name="dense-and-sparse, 13B shapes, 0.45% fp16 CSR", shapes=LLAMA2_13B,
                        Ms=[1, 16, 1024], csr=True)
LARGE_LAYERS_70B = dict(family=4, name="large layers, 70B shapes", shapes=LLAMA2_70B, Ms=[1, 64, 4096], csr=False)
WORKLOADS = (SINGLE_LAYER, DECODE_SWEEP, PREFILL_SWEEP, DENSE_SPARSE_13B, LARGE_LAYERS_70B)
ALPHA = 0.5
OUTLIER_FRACTION = 0.0045
N_OUTLIER_CHANNELS = 8
OUTLIER_CHANNEL_GAIN = 20.0
CALIB_ROWS = 512


def seed_of(family: int, shape_index: int) -> int:
    return 1000 * family + shape_index


def _streams(seed: int):
    ss = np.random.SeedSequence(seed)
    return [np.random.Generator(np.random.PCG64(c)) for c in ss.spawn(5)]


@dataclass
class Layer:
    K: int
    N: int
    W: np.ndarray            # fp32 [N][K]
    mult: np.ndarray         # fp32 [K] per-channel activation multipliers m_k
    act_absmean: np.ndarray  # fp32 [K]
    seed: int


def make_layer(seed: int, K: int, N: int, calib_rows: int = CALIB_ROWS) -> Layer:
    rw, rm, ro, rc, _ = _streams(seed)
    W = rw.standard_normal((N, K), dtype=np.float32)
    W *= np.float32(0.02)
    mult = np.exp(rm.standard_normal(K)).astype(np.float64)
    idx = ro.choice(K, size=min(N_OUTLIER_CHANNELS, K), replace=False)
    mult[idx] *= OUTLIER_CHANNEL_GAIN
    # |X_cal| mean over the calibration rows, in fp64, in chunks to bound memory
    acc = np.zeros(K, np.float64)
    done = 0
    while done < calib_rows:
        r = min(64, calib_rows - done)
        acc += np.abs(rc.standard_normal((r, K)) * mult).sum(axis=0)
        done += r
    act = (acc / calib_rows).astype(np.float32)
    return Layer(K=K, N=N, W=W, mult=mult.astype(np.float32), act_absmean=act, seed=seed)


def make_act_absmean(seed: int, K: int, calib_rows: int = CALIB_ROWS):
    """(mult, act_absmean) of make_layer(seed, K, N) without drawing W (for layers too large to
    draw on the host; the same substreams, so the values equal make_layer's)."""
    _, rm, ro, rc, _ = _streams(seed)
    mult = np.exp(rm.standard_normal(K)).astype(np.float64)
    idx = ro.choice(K, size=min(N_OUTLIER_CHANNELS, K), replace=False)
    mult[idx] *= OUTLIER_CHANNEL_GAIN
    acc = np.zeros(K, np.float64)
    done = 0
    while done < calib_rows:
        r = min(64, calib_rows - done)
        acc += np.abs(rc.standard_normal((r, K)) * mult).sum(axis=0)
        done += r
    return mult.astype(np.float32), (acc / calib_rows).astype(np.float32)


def _f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest-even) via torch's conversion; returns uint16 bits."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def make_activations(seed: int, M: int, mult: np.ndarray, alpha: float = ALPHA) -> np.ndarray:
    """x' bf16 bits [M][K] = bf16(N(0,1) * m_k^(1-alpha)); rows are a prefix of one stream."""
    _, _, _, _, rx = _streams(seed)
    K = mult.size
    z = rx.standard_normal((M, K)).astype(np.float32)
    spread = np.power(mult.astype(np.float64), 1.0 - alpha).astype(np.float32)
    return _f32_to_bf16_bits(z * spread)


def uniform_bf16(seed: int, shape, lo=-1.0, hi=1.0) -> np.ndarray:
    """Plain uniform bf16 bits (for edge-case tests that need no particular structure)."""
    r = np.random.Generator(np.random.PCG64(seed))
    return _f32_to_bf16_bits(r.uniform(lo, hi, size=shape).astype(np.float32))


def outlier_nnz(N: int, K: int, fraction: float = OUTLIER_FRACTION) -> int:
    """Number of entries the dense-and-sparse split keeps in fp16: floor(fraction * N * K)."""
    return int(np.floor(fraction * N * K))


def packed_bytes(N: int, K: int) -> int:
    """Bytes of the packed weight set (qweight + fp16 scales + zeros) for an N x K layer."""
    return N * K // 2 + N * (K // 128) * 2 + N * (K // 1024) * 4
