"""The five synthetic workloads (parameter-shaped stand-ins; no dataset).

1  one flat tensor, n = 1,048,576, N(0, 1e-3) from seed 0, s = 1.0, one step.
2  ResNet-110 (CIFAR, option-A shortcuts) 3x3 conv weights: 109 tensors,
   1,719,216 values, N(0, 1e-3) with 60% iid exact zeros, s = 1.75, 20 steps
   with the error buffer carried per tensor.
3  one flat tensor of 2^28 values (and a sweep 2^20..2^28), Laplace(0, 1e-4)
   with 90% exact zeros in alternating runs (zero runs geometric with mean 64,
   non-zero runs geometric with mean 64/9, a zero run first), s = 1.9.
4  BERT-large parameter set: 391 tensors, 335,141,888 values, N(0, 1e-3);
   the 30522 x 1024 word embedding has each row all-zero with p = 0.99;
   s = 1.5, 5 steps with error feedback.
5  K = 8 worker streams of one ResNet-50-sized bucket (25,557,032 values),
   N(0, 1e-3), worker seeds 0..7, s = 1.75, decoded and summed.

The second parameter of N(.,.) is the standard deviation and of Laplace(.,.)
the scale b.  The seed of tensor t at step k is
base XOR splitmix64(k * 2^20 + t); values and masks use separate streams.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor

import numpy as np

from .gen import (bernoulli, key_for, laplace, normal, splitmix64_mix,
                  zero_runs_mask)

P_VALUES, P_MASK, P_RUNS = 0, 3, 4


def tensor_seed(base: int, step: int, idx: int) -> int:
    return (int(base) ^ int(splitmix64_mix(np.uint64(step * (1 << 20) + idx)))) & ((1 << 64) - 1)


def resnet110_conv_shapes():
    """(out, in, 3, 3) of the 109 conv layers of CIFAR ResNet-110."""
    shapes = [(16, 3, 3, 3)]
    for cin, cout in ((16, 16), (16, 32), (32, 64)):
        for blk in range(18):
            first_in = cin if blk == 0 else cout
            shapes.append((cout, first_in, 3, 3))
            shapes.append((cout, cout, 3, 3))
    return shapes


def bert_large_shapes():
    """Parameter shapes of BERT-large (24 layers, hidden 1024, FFN 4096)."""
    h, f, v = 1024, 4096, 30522
    shapes = [(v, h), (512, h), (2, h), (h,), (h,)]
    for _ in range(24):
        for _qkvo in range(4):
            shapes += [(h, h), (h,)]
        shapes += [(h,), (h,)]              # attention output LayerNorm
        shapes += [(h, f), (f,), (f, h), (h,)]
        shapes += [(h,), (h,)]              # output LayerNorm
    shapes += [(h, h), (h,)]                # pooler
    return shapes


CONFIGS = {
    1: dict(name="flat 2^20 N(0,1e-3), s=1.0", s=1.0, steps=1, n=1_048_576),
    2: dict(name="ResNet-110 conv set (109 tensors), 60% zeros, s=1.75",
            s=1.75, steps=20),
    3: dict(name="flat 2^28 Laplace(0,1e-4), 90% zeros in geometric runs, s=1.9",
            s=1.9, steps=1, n=1 << 28),
    4: dict(name="BERT-large set (391 tensors), embedding rows 99% zero, s=1.5",
            s=1.5, steps=5),
    5: dict(name="K=8 streams of 25,557,032 values, N(0,1e-3), s=1.75",
            s=1.75, steps=1, n=25_557_032, k=8),
}


def _numel(shape):
    return int(np.prod(shape))


def flat_tensor(cfg: int, n: int | None = None, step: int = 0, worker: int = 0) -> np.ndarray:
    """The gradient of config 1, 3 or 5 (worker = stream index for config 5)."""
    c = CONFIGS[cfg]
    n = int(c["n"] if n is None else n)
    if cfg == 1:
        return normal(key_for(tensor_seed(0, step, 0), P_VALUES), n, 1e-3)
    if cfg == 3:
        seed = tensor_seed(0, step, 0)
        x = laplace(key_for(seed, P_VALUES), n, 1e-4)
        x[zero_runs_mask(key_for(seed, P_RUNS), n, 64.0, 64.0 / 9.0)] = 0.0
        return x
    if cfg == 5:
        return normal(key_for(tensor_seed(worker, step, 0), P_VALUES), n, 1e-3)
    raise ValueError(f"config {cfg} is a tensor set")


def tensor_set(cfg: int, step: int, limit: int | None = None):
    """The per-layer gradients of config 2 or 4 at `step` (first `limit`)."""
    if cfg == 2:
        shapes = resnet110_conv_shapes()
    elif cfg == 4:
        shapes = bert_large_shapes()
    else:
        raise ValueError(f"config {cfg} is a flat tensor")
    todo = list(enumerate(shapes[:limit] if limit else shapes))

    def one(item):
        t, shp = item
        seed = tensor_seed(0, step, t)
        n = _numel(shp)
        x = normal(key_for(seed, P_VALUES), n, 1e-3)
        if cfg == 2:
            x[bernoulli(key_for(seed, P_MASK), n, 0.6)] = 0.0
        elif t == 0:   # word embedding: whole rows zero with p = 0.99
            rows = bernoulli(key_for(seed, P_MASK), shp[0], 0.99)
            x.reshape(shp)[rows, :] = 0.0
        return x

    # tensors are independent; a separate pool from the chunk pool in gen.py
    with ThreadPoolExecutor(4) as pool:
        return list(pool.map(one, todo))


def config_step_inputs(cfg: int, step: int = 0):
    """All gradients of one step of a config, as a list of fp32 arrays."""
    if cfg in (2, 4):
        return tensor_set(cfg, step)
    if cfg == 5:
        return [flat_tensor(5, step=step, worker=w) for w in range(CONFIGS[5]["k"])]
    return [flat_tensor(cfg, step=step)]
