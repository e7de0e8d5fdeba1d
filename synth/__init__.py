"""Seeded synthetic gradient generator shared by the tests and the benchmark.

It holds none of the compression method's arithmetic, only random inputs.
Every value comes from a counter-based generator: splitmix64 (Steele, Lea and
Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014) applied
to key + i * 0x9E3779B97F4A7C15.  Uniforms are (top 53 bits + 0.5) * 2^-53,
in (0, 1).  Distributions are formed in float64 and cast to fp32 last:

* normal(sigma): Box-Muller from two uniforms, cosine branch only;
* laplace(b): inverse CDF, -b * sign(u - 1/2) * ln(1 - 2|u - 1/2|);
* Bernoulli(p) masks: u < p;
* geometric run lengths of mean mu (support >= 1): 1 + floor(ln u / ln(1 - 1/mu)).

The integer layer is deterministic everywhere; the float layer uses numpy's
log/cos/sqrt and may differ in the last bit between machines, so no stored
expected value is ever derived from it.
"""
from .gen import (  # noqa: F401
    GOLDEN_RATIO64,
    splitmix64_mix,
    key_for,
    uniforms,
    normal,
    laplace,
    bernoulli,
    geometric,
    zero_runs_mask,
)
from .configs import (  # noqa: F401
    CONFIGS,
    resnet110_conv_shapes,
    bert_large_shapes,
    tensor_set,
    flat_tensor,
    config_step_inputs,
)
